"""The C-ABI library: it loads, exports every symbol include/gdn.h declares,
and rejects bad arguments on the host before launching anything.

The argument-error cases pass fake device pointers; they only run where no
CUDA device is present, so that a validation bug can never hand a kernel a
bogus address.
"""
import ctypes
import os
import re

import pytest

import linear_attention_layer_causal_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"GDN_API\s+[\w\s\*]*?\b(gdn_\w+)\s*\(", txt)
    return names


def test_library_exports_every_declared_symbol():
    L = gdn.lib()
    declared = _declared()
    assert set(gdn.EXPORTED) <= set(declared)
    for name in declared:
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
    assert L.gdn_abi_version() == 3


def test_status_strings():
    for s in range(6):
        assert gdn.status_string(s)
    assert "wait" in gdn.status_string(gdn.GDN_ERR_TIMEOUT)
    assert gdn.status_string(99) == "unknown status"


QWEN38 = gdn.Config(16, 128, 128)


def test_workspace_size_arithmetic():
    n = gdn.prefill_workspace_size(QWEN38, 1, 4096)
    # 256-byte header (status word), float32 normalised q|k and, on the chunked
    # path, the chunks' Q K^T rows [N, H_k, 64], K K^T tiles [N / 64 + batch
    # chunks, H_k, 3072], T diag(beta) and -T diag(beta gamma) tiles [chunks, H_v,
    # 2, 96, 32], gate records [chunks, H_v, 3, 64] and the chunk offsets [batch +
    # 1]; regions rounded to 256 B.  With 16-bit activations the chunk kernel
    # convolves v itself: no float32 v
    tile = 2 * 128 * 96 * 32 * 4 + 16 * 3072 * 4 + 128 * 192 * 4  # one chunk's tiles, all heads
    assert n == (256 + 4096 * 2 * 16 * 128 * 4 + 4096 * 16 * 64 * 4 + (64 + 1) * tile + 256)
    # float32 activations add the convolved v [N, H_v * 128]
    assert gdn.prefill_workspace_size(gdn.Config(16, 128, 128, act_dtype="f32"), 1, 4096) == \
        n + 4096 * 128 * 128 * 4
    # the token-serial path: header, q|k and v only
    assert gdn.prefill_workspace_size(gdn.Config(16, 128, 128, algo="serial"), 1, 4096) == \
        256 + 4096 * 2 * 16 * 128 * 4 + 4096 * 128 * 128 * 4
    # 99 more sequences: at most 99 more (partial) chunks, and 512 bytes of offsets
    assert gdn.prefill_workspace_size(QWEN38, 100, 4096) == n + 99 * tile + 256
    assert gdn.prefill_workspace_size(QWEN38, 0, 0) == 0
    # sequences but no tokens: nothing for a kernel to stage, and no workspace (the
    # launches that would need one -- chunk offsets, status words -- are skipped)
    assert gdn.prefill_workspace_size(QWEN38, 3, 0) == 0
    assert gdn.prefill_workspace_size(gdn.Config(2, 4, 32), 5, 0) == 0
    tiny = gdn.Config(2, 4, 32, act_dtype="f32")
    assert gdn.prefill_workspace_size(tiny, 1, 3) == 256 + 1536 + 1536
    assert gdn.prefill_workspace_size(tiny, 1, 1) == 256 + 512 + 512
    assert gdn.prefill_workspace_size(gdn.Config(2, 4, 32), 1, 3) == 256 + 1536 + 1536


def test_kda_workspace_size_arithmetic():
    """KDA prefill: a 256-byte header, float32 normalised q|k [N, 2 H d], float32
    convolved v [N, H d] and the float32 raw output [N, H, d] that the recurrence
    writes and the gated-norm pass reads; regions rounded to 256 B."""
    kimi = gdn.Config(96, 96, 128)
    N = 4096
    assert gdn.kda_prefill_workspace_size(kimi, 1, N) == 256 + N * 2 * 96 * 128 * 4 + 2 * N * 96 * 128 * 4
    # the size does not depend on the sequence count, and no tokens need none
    assert gdn.kda_prefill_workspace_size(kimi, 7, N) == gdn.kda_prefill_workspace_size(kimi, 1, N)
    assert gdn.kda_prefill_workspace_size(kimi, 3, 0) == 0
    small = gdn.Config(4, 4, 32, act_dtype="f32")
    # 3 tokens: q|k 3 * 2 * 4 * 32 * 4 = 3072 B, v and o 1536 B each
    assert gdn.kda_prefill_workspace_size(small, 2, 3) == 256 + 3072 + 1536 + 1536
    # 1 token: 1024 B, then 512 B each
    assert gdn.kda_prefill_workspace_size(small, 1, 1) == 256 + 1024 + 512 + 512
    # KDA has one q/k head per value head and no sequence split
    for bad in (gdn.Config(2, 4, 32), gdn.Config(4, 4, 32, segments=2)):
        with pytest.raises(gdn.GdnError):
            gdn.kda_prefill_workspace_size(bad, 1, 8)


def test_segment_workspace_and_choice():
    """The split's workspace (R, M and start states: 3 (P - 1) batch H_v d^2 floats)
    and the library's choice of P."""
    state = 128 * 128 * 4
    for B, N in ((1, 4096), (3, 20000)):
        base = gdn.prefill_workspace_size(gdn.Config(16, 128, 128, segments=1), B, N)
        assert gdn.prefill_workspace_size(QWEN38, B, N) == base  # 128 value heads: no split
        for P in (2, 5, 16):
            c = gdn.Config(16, 128, 128, segments=P)
            assert gdn.prefill_workspace_size(c, B, N) == base + 3 * (P - 1) * B * 128 * state
    # the token-serial path takes segments 0 and 1
    for P in (0, 1):
        assert gdn.prefill_workspace_size(gdn.Config(2, 4, 32, segments=P), 1, 3) == 256 + 1536 + 1536
    # no tokens: no workspace, whatever P
    assert gdn.prefill_workspace_size(gdn.Config(16, 128, 128, segments=4), 2, 0) == 0
    # the library's choice at 64 value heads: one sequence of 262,144 tokens is split
    # (64 chains would leave 84 of the 148 SMs idle), one of 2,048 is not (too short),
    # and neither is a batch of 2 x 131,072 (128 chains fill the SMs)
    q35 = gdn.Config(16, 64, 128)
    one = gdn.Config(16, 64, 128, segments=1)
    extra = gdn.prefill_workspace_size(q35, 1, 262144) - gdn.prefill_workspace_size(one, 1, 262144)
    assert extra > 0 and extra % (3 * 64 * state) == 0
    assert gdn.prefill_workspace_size(q35, 1, 2048) == gdn.prefill_workspace_size(one, 1, 2048)
    assert gdn.prefill_workspace_size(q35, 2, 262144) == gdn.prefill_workspace_size(one, 2, 262144)
    assert gdn.prefill_segments(q35, 1, 262144) == 1 + extra // (3 * 64 * state)
    assert gdn.prefill_segments(QWEN38, 1, 262144) == 1
    assert gdn.prefill_segments(gdn.Config(16, 128, 128, segments=7), 1, 100) == 7
    assert gdn.prefill_segments(gdn.Config(16, 128, 128, segments=7), 1, 0) == 1
    assert gdn.prefill_segments(gdn.Config(2, 4, 32), 1, 1 << 20) == 1
    # few heads, a long sequence: several segments
    small = gdn.Config(2, 8, 128)
    extra = (gdn.prefill_workspace_size(small, 1, 1 << 20) -
             gdn.prefill_workspace_size(gdn.Config(2, 8, 128, segments=1), 1, 1 << 20))
    assert extra // (3 * 8 * state) + 1 >= 4


@pytest.mark.parametrize("cfg,code", [
    (gdn.Config(0, 4, 32), gdn.GDN_ERR_INVALID_ARG),
    (gdn.Config(3, 4, 32), gdn.GDN_ERR_INVALID_ARG),        # H_v not a multiple of H_k
    (gdn.Config(2, 4, 64), gdn.GDN_ERR_UNSUPPORTED),        # head dim without a kernel
    (gdn.Config(2, 4, 32, conv_kernel=3), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.Config(2, 4, 32, rms_eps=-1.0), gdn.GDN_ERR_INVALID_ARG),
    (gdn.Config(2, 4, 32, l2_eps=float("nan")), gdn.GDN_ERR_INVALID_ARG),
    (gdn.Config(2, 4, 32, algo="chunked"), gdn.GDN_ERR_UNSUPPORTED),  # chunked needs d = 128
    (gdn.Config(16, 128, 128, segments=-1), gdn.GDN_ERR_INVALID_ARG),
    (gdn.Config(16, 128, 128, segments=17), gdn.GDN_ERR_INVALID_ARG),
    (gdn.Config(2, 4, 32, segments=2), gdn.GDN_ERR_UNSUPPORTED),      # the split is chunked-only
    (gdn.Config(16, 128, 128, algo="serial", segments=2), gdn.GDN_ERR_UNSUPPORTED),
])
def test_bad_config_rejected(cfg, code):
    n = ctypes.c_size_t(0)
    assert gdn.lib().gdn_prefill_workspace_size(ctypes.byref(cfg._c()), 1, 10, ctypes.byref(n)) == code


def test_unknown_algo_rejected():
    c = gdn.Config(2, 4, 32)._c()
    c.algo = 3
    n = ctypes.c_size_t(0)
    assert gdn.lib().gdn_prefill_workspace_size(ctypes.byref(c), 1, 10, ctypes.byref(n)) == \
        gdn.GDN_ERR_INVALID_ARG


def _fake_call(**over):
    """gdn_prefill with fake 256-aligned device pointers; `over` replaces arguments."""
    cfg = over.pop("cfg", gdn.Config(2, 4, 32))
    P = 1 << 20
    par = gdn._Params(P, P + 256, P + 512, P + 768)
    args = dict(qkv=P * 2, a=P * 3, b=P * 4, z=P * 5, cu=P * 6, batch=1, N=10, S0=None,
                C0=None, y=P * 7, S1=None, C1=None, o=None, ws=P * 8, wsb=1 << 20)
    args.update(over)
    params = over.get("params", par)
    return gdn.lib().gdn_prefill(ctypes.byref(cfg._c()), ctypes.byref(params), args["qkv"],
                                 args["a"], args["b"], args["z"], args["cu"], args["batch"],
                                 args["N"], args["S0"], args["C0"], args["y"], args["S1"],
                                 args["C1"], args["o"], args["ws"], args["wsb"], None)


no_gpu = pytest.mark.skipif(
    __import__("torch").cuda.is_available(), reason="argument-error cases run only without a GPU")


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(qkv=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(y=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(qkv=(1 << 21) + 8), gdn.GDN_ERR_INVALID_ARG),     # 8-byte aligned only
    (dict(S0=(1 << 22) + 4), gdn.GDN_ERR_INVALID_ARG),
    (dict(a=(1 << 22) + 1), gdn.GDN_ERR_INVALID_ARG),       # odd address for bf16
    (dict(batch=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-5), gdn.GDN_ERR_INVALID_ARG),
    (dict(batch=0, N=10), gdn.GDN_ERR_INVALID_ARG),
    (dict(batch=70000), gdn.GDN_ERR_UNSUPPORTED),
    (dict(ws=None), gdn.GDN_ERR_WORKSPACE),
    (dict(wsb=100), gdn.GDN_ERR_WORKSPACE),
    (dict(ws=(1 << 23) + 16), gdn.GDN_ERR_WORKSPACE),       # not 256-byte aligned
    (dict(params=gdn._Params(None, 256, 512, 768)), gdn.GDN_ERR_INVALID_ARG),
    (dict(params=gdn._Params(8, 256, 512, 768)), gdn.GDN_ERR_INVALID_ARG),
    (dict(cfg=gdn.Config(2, 4, 48)), gdn.GDN_ERR_UNSUPPORTED),
    # the chunked path's tile rows (192 per chunk and value head) exceed 32-bit
    # TMA coordinates; the token-serial path has no such tiles
    (dict(cfg=gdn.Config(16, 128, 128), N=6_000_000), gdn.GDN_ERR_UNSUPPORTED),
    (dict(cfg=gdn.Config(16, 128, 128, algo="serial"), N=6_000_000), gdn.GDN_ERR_WORKSPACE),
])
def test_prefill_argument_errors(over, code):
    assert _fake_call(**over) == code


@no_gpu
def test_decode_argument_errors():
    L = gdn.lib()
    cfg = gdn.Config(2, 4, 32)
    par = gdn._Params(1 << 20, (1 << 20) + 256, (1 << 20) + 512, (1 << 20) + 768)
    P = 1 << 24
    ok = [P, P * 2, P * 3, P * 4, P * 5, P * 6, 3, P * 7, None]
    def call(i, v):
        a = list(ok)
        a[i] = v
        return L.gdn_decode(ctypes.byref(cfg._c()), ctypes.byref(par), *a)
    assert call(4, None) == gdn.GDN_ERR_INVALID_ARG          # state
    assert call(5, None) == gdn.GDN_ERR_INVALID_ARG          # conv cache
    assert call(4, P + 8) == gdn.GDN_ERR_INVALID_ARG         # misaligned state
    assert call(6, -1) == gdn.GDN_ERR_INVALID_ARG
    assert call(6, 0) == gdn.GDN_OK                          # empty batch: nothing to do
    assert L.gdn_decode(None, ctypes.byref(par), *ok) == gdn.GDN_ERR_INVALID_ARG


@no_gpu
def test_multi_token_decode_argument_errors():
    L = gdn.lib()
    cfg = gdn.Config(16, 128, 128)
    par = gdn._Params(1 << 20, (1 << 20) + 256, (1 << 20) + 512, (1 << 20) + 768)
    P = 1 << 24
    c, p_ = ctypes.byref(cfg._c()), ctypes.byref(par)
    # qkv, a, b, z, state, conv_cache, batch, k, y
    ok = [P, P * 2, P * 3, P * 4, P * 5, P * 6, 3, 2, P * 7, None]
    assert L.gdn_decode_multi(c, p_, *ok[:7], 0, *ok[8:]) == gdn.GDN_ERR_INVALID_ARG   # k = 0
    assert L.gdn_decode_multi(c, p_, *ok[:7], 9, *ok[8:]) == gdn.GDN_ERR_UNSUPPORTED   # k > 8
    assert L.gdn_decode_verify(c, p_, *ok[:8], None, None) == gdn.GDN_ERR_INVALID_ARG  # no y
    assert L.gdn_decode_multi(c, p_, *ok[:7], 2, P * 7 + 8, None) == gdn.GDN_ERR_INVALID_ARG
    # commit: qkv, a, b, state, conv_cache, batch, k, accepted
    assert L.gdn_decode_commit(c, p_, P, P * 2, P * 3, P * 5, P * 6, 3, 2, None, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_decode_commit(c, p_, P, P * 2, P * 3, P * 5, P * 6, 3, 2, P * 8 + 2, None) == \
        gdn.GDN_ERR_INVALID_ARG                                                      # misaligned
    assert L.gdn_decode_commit(c, p_, P, P * 2, P * 3, P * 5, P * 6, 0, 2, None, None) == \
        gdn.GDN_OK                                                                   # no sequences
    # G = 64 at d = 128: k = 8 tokens of a group need more shared memory than a CTA has
    wide = gdn.Config(1, 64, 128)
    assert L.gdn_decode_multi(ctypes.byref(wide._c()), p_, *ok[:7], 8, *ok[8:]) == \
        gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_decode_multi(ctypes.byref(wide._c()), p_, *ok[:6], 0, 2, *ok[8:]) == gdn.GDN_OK


@no_gpu
def test_noalloc_rejects_oversized_calls_on_the_host():
    """The fixed-scratch prefill refuses, before any CUDA call, a call that needs
    more than GDN_NOALLOC_SCRATCH_BYTES of scratch."""
    L = gdn.lib()
    cfg = gdn.Config(16, 128, 128)
    P = 1 << 20
    par = gdn._Params(P, P + 256, P + 512, P + 768)
    n_big = 2000
    assert gdn.prefill_workspace_size(cfg, 1, n_big) > gdn.NOALLOC_SCRATCH_BYTES
    args = [P * 2, P * 3, P * 4, P * 5, P * 6, 1, n_big, None, None, P * 7, None, None, None, None]
    assert L.gdn_prefill_noalloc(ctypes.byref(cfg._c()), ctypes.byref(par), *args) == \
        gdn.GDN_ERR_WORKSPACE
    bad = gdn.Config(3, 4, 32)
    assert L.gdn_prefill_noalloc(ctypes.byref(bad._c()), ctypes.byref(par), *args) == \
        gdn.GDN_ERR_INVALID_ARG


@no_gpu
def test_noalloc_checks_arguments_before_the_scratch_size():
    """gdn_prefill_noalloc validates like gdn_prefill (same codes, same order) and only
    then refuses a call that is too large for its fixed scratch."""
    L = gdn.lib()
    cfg = gdn.Config(16, 128, 128)
    P = 1 << 20
    par = gdn._Params(P, P + 256, P + 512, P + 768)
    big = [P * 2, P * 3, P * 4, P * 5, P * 6, 1, 100000, None, None, P * 7, None, None, None,
           None]
    bad_qkv = list(big)
    bad_qkv[0] = None
    assert L.gdn_prefill_noalloc(ctypes.byref(cfg._c()), ctypes.byref(par), *bad_qkv) == \
        gdn.GDN_ERR_INVALID_ARG
    misaligned = list(big)
    misaligned[9] = P * 7 + 8  # y only 8-byte aligned
    assert L.gdn_prefill_noalloc(ctypes.byref(cfg._c()), ctypes.byref(par), *misaligned) == \
        gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_prefill_noalloc(ctypes.byref(cfg._c()), ctypes.byref(par), *big) == \
        gdn.GDN_ERR_WORKSPACE


def test_status_query_and_wait_limit_argument_errors():
    L = gdn.lib()
    d = ctypes.c_uint32(7)
    assert L.gdn_prefill_status(None, 1 << 20, ctypes.byref(d), None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_prefill_status(1 << 20, 4, ctypes.byref(d), None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_wait_limit_next_call(-1) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_wait_limit_next_call(0) == gdn.GDN_OK  # disarmed


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "LIB_PATH", str(tmp_path / "libgdn.so"))
    with pytest.raises(RuntimeError, match="missing"):
        gdn.lib()
