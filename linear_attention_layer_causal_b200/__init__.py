"""B200 (sm_100a) Gated DeltaNet token mixer.

Thin ctypes binding over ``libgdn.so`` (C ABI in ``include/gdn.h``).  This
module only marshals arguments: it turns torch tensors into device pointers
and the current CUDA stream into a ``cudaStream_t``, allocates outputs and
workspace with torch, and raises on a non-zero status.  Every step of the
layer runs in the library's CUDA kernels; there is no CPU path, and calling
into the library without the built extension raises.

    import linear_attention_layer_causal_b200 as gdn
    cfg = gdn.Config(num_qk_heads=16, num_v_heads=128, head_dim=128)
    out = gdn.prefill(cfg, qkv, a, b, z, cu_seqlens, conv_w, A_log, dt_bias, norm_w,
                      initial_state=S0, return_final_state=True)
    y = gdn.decode(cfg, qkv1, a1, b1, z1, state, conv_cache, conv_w, A_log, dt_bias, norm_w)

The layer: kernel-4 causal conv + SiLU over q|k|v, q/k L2 norm, gates
g = -exp(A_log) softplus(a + dt_bias) and beta = sigmoid(b), the gated delta
rule on an FP32 state per value head, and the per-head RMSNorm gated by
SiLU(z) (Gated DeltaNet and output-gate rows of the component table on
"Qwen3.8-2.4T-A95B vs Inkling").
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

(GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA,
 GDN_ERR_TIMEOUT) = range(6)
GDN_F32, GDN_BF16 = 0, 1

EXPORTED = ("gdn_prefill_workspace_size", "gdn_prefill_segments", "gdn_prefill", "gdn_decode", "gdn_status_string",
            "gdn_abi_version", "gdn_profile_next_call", "gdn_prefill_noalloc",
            "gdn_prefill_status", "gdn_prefill_noalloc_status", "gdn_wait_limit_next_call",
            "gdn_decode_multi", "gdn_decode_verify", "gdn_decode_commit",
            "gdn_kda_prefill_workspace_size", "gdn_kda_prefill", "gdn_kda_decode")

# Fixed scratch of gdn_prefill_noalloc (GDN_NOALLOC_SCRATCH_BYTES in include/gdn.h).
NOALLOC_SCRATCH_BYTES = 64 << 20


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


class _Config(ctypes.Structure):
    _fields_ = [("num_qk_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("conv_kernel", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("l2_eps", ctypes.c_float),
                ("q_scale", ctypes.c_float), ("act_dtype", ctypes.c_int32),
                ("algo", ctypes.c_int32), ("segments", ctypes.c_int32)]


class _KdaParams(ctypes.Structure):
    _fields_ = [("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
                ("norm_w", ctypes.c_void_p)]


class _Params(ctypes.Structure):
    _fields_ = [("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p), ("norm_w", ctypes.c_void_p)]


@dataclass(frozen=True)
class Config:
    """Head layout of one layer (H_k q/k heads, H_v value heads, head dim d)."""
    num_qk_heads: int
    num_v_heads: int
    head_dim: int
    conv_kernel: int = 4
    rms_eps: float = 1e-6
    l2_eps: float = 1e-6
    q_scale: float = 1.0
    act_dtype: str = "bf16"  # "bf16" or "f32"
    algo: str = "auto"       # prefill algorithm: "auto", "serial" or "chunked"
    segments: int = 0        # chunked prefill: segments per sequence (0 = the library's choice)

    @property
    def conv_dim(self) -> int:
        return (2 * self.num_qk_heads + self.num_v_heads) * self.head_dim

    def _c(self) -> _Config:
        return _Config(self.num_qk_heads, self.num_v_heads, self.head_dim, self.conv_kernel,
                       self.rms_eps, self.l2_eps, self.q_scale,
                       GDN_BF16 if self.act_dtype == "bf16" else GDN_F32,
                       {"auto": 0, "serial": 1, "chunked": 2}[self.algo], self.segments)

    @staticmethod
    def of(wl, algo: str = "auto", segments: int = 0) -> "Config":
        """The Config of a workloads.Workload."""
        return Config(wl.num_qk_heads, wl.num_v_heads, wl.head_dim, wl.conv_kernel,
                      act_dtype=wl.dtype, algo=algo, segments=segments)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m linear_attention_layer_causal_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        cfgp, parp = ctypes.POINTER(_Config), ctypes.POINTER(_Params)
        L.gdn_prefill_workspace_size.argtypes = [cfgp, i32, i64, ctypes.POINTER(sz)]
        L.gdn_prefill_workspace_size.restype = ctypes.c_int
        L.gdn_prefill_segments.argtypes = [cfgp, i32, i64, ctypes.POINTER(i32)]
        L.gdn_prefill_segments.restype = ctypes.c_int
        L.gdn_prefill.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp, vp,
                                  vp, vp, sz, vp]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill_noalloc.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp,
                                          vp, vp, vp, vp]
        L.gdn_prefill_noalloc.restype = ctypes.c_int
        L.gdn_decode.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_decode_multi.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.gdn_decode_multi.restype = ctypes.c_int
        L.gdn_decode_verify.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.gdn_decode_verify.restype = ctypes.c_int
        L.gdn_decode_commit.argtypes = [cfgp, parp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.gdn_decode_commit.restype = ctypes.c_int
        kpp = ctypes.POINTER(_KdaParams)
        L.gdn_kda_prefill_workspace_size.argtypes = [cfgp, i32, i64, ctypes.POINTER(sz)]
        L.gdn_kda_prefill_workspace_size.restype = ctypes.c_int
        L.gdn_kda_prefill.argtypes = [cfgp, kpp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp, vp,
                                      vp, vp, sz, vp]
        L.gdn_kda_prefill.restype = ctypes.c_int
        L.gdn_kda_decode.argtypes = [cfgp, kpp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
        L.gdn_kda_decode.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_profile_next_call.argtypes = [vp, vp]
        L.gdn_profile_next_call.restype = ctypes.c_int
        u32p = ctypes.POINTER(ctypes.c_uint32)
        L.gdn_prefill_status.argtypes = [vp, sz, u32p, vp]
        L.gdn_prefill_status.restype = ctypes.c_int
        L.gdn_prefill_noalloc_status.argtypes = [u32p, vp]
        L.gdn_prefill_noalloc_status.restype = ctypes.c_int
        L.gdn_wait_limit_next_call.argtypes = [i64]
        L.gdn_wait_limit_next_call.restype = ctypes.c_int
        L.gdn_abi_version.argtypes = []
        L.gdn_abi_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(status).decode()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _act(cfg: Config):
    import torch
    return torch.bfloat16 if cfg.act_dtype == "bf16" else torch.float32


def _params(conv_w, A_log, dt_bias, norm_w) -> _Params:
    return _Params(_ptr(conv_w), _ptr(A_log), _ptr(dt_bias), _ptr(norm_w))


def profile_next_call(begin_event, end_event) -> None:
    """Time the main kernel of this thread's next prefill/decode call between two
    torch.cuda.Event(enable_timing=True) events (see gdn_profile_next_call)."""
    for ev in (begin_event, end_event):
        if ev is not None and not ev.cuda_event:
            ev.record()  # torch creates the underlying cudaEvent_t on first record
    b = None if begin_event is None else begin_event.cuda_event
    e = None if end_event is None else end_event.cuda_event
    st = lib().gdn_profile_next_call(b, e)
    if st != GDN_OK:
        raise GdnError(st, "gdn_profile_next_call")


def prefill_status(workspace, stream=None) -> tuple[int, int]:
    """(status, detail) of the last prefill that used `workspace` (gdn_prefill_status):
    GDN_OK, GDN_ERR_TIMEOUT when a bounded wait inside a kernel gave up, or
    GDN_ERR_CUDA; detail says where the first timed-out wait gave up.  Waits for
    the stream."""
    if workspace is None or workspace.numel() < 8:
        return GDN_OK, 0
    d = ctypes.c_uint32(0)
    st = lib().gdn_prefill_status(_ptr(workspace), workspace.numel(), ctypes.byref(d),
                                  _stream(stream))
    return st, d.value


def prefill_noalloc_status(stream=None) -> tuple[int, int]:
    """(status, detail) of the last gdn_prefill_noalloc call on the current device."""
    d = ctypes.c_uint32(0)
    st = lib().gdn_prefill_noalloc_status(ctypes.byref(d), _stream(stream))
    return st, d.value


def wait_limit_next_call(cycles: int) -> None:
    """Testing hook: the next prefill call on this thread bounds each wait between
    the warps of its chunked kernel by `cycles` SM cycles (0 = default, ~1 s)."""
    st = lib().gdn_wait_limit_next_call(int(cycles))
    if st != GDN_OK:
        raise GdnError(st, "gdn_wait_limit_next_call")


def prefill_workspace_size(cfg: Config, batch: int, total_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    st = lib().gdn_prefill_workspace_size(ctypes.byref(cfg._c()), batch, total_tokens,
                                          ctypes.byref(n))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill_workspace_size")
    return n.value


def prefill_segments(cfg: Config, batch: int, total_tokens: int) -> int:
    """Segments per sequence a prefill of this size runs with (gdn_prefill_segments)."""
    n = ctypes.c_int32(0)
    st = lib().gdn_prefill_segments(ctypes.byref(cfg._c()), batch, total_tokens, ctypes.byref(n))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill_segments")
    return n.value


def prefill(cfg: Config, qkv, a, b, z, cu_seqlens, conv_w, A_log, dt_bias, norm_w, *,
            initial_state=None, initial_conv=None, return_final_state=False,
            return_final_conv=False, return_o_raw=False, y=None, final_state=None,
            final_conv=None, workspace=None, stream=None, check_status=False) -> dict:
    """Packed varlen prefill (see gdn_prefill in include/gdn.h).

    Returns a dict with "y" and, when requested, "final_state", "final_conv"
    and "o_raw".  Output buffers and the workspace may be passed in to avoid
    allocation; ``final_state`` may be ``initial_state`` for an in-place update.
    With ``check_status`` the call synchronises and raises if a kernel reported
    a failure in the workspace status word.
    """
    import torch
    N = qkv.shape[0]
    B = cu_seqlens.shape[0] - 1
    dev = qkv.device
    if y is None:
        y = torch.empty((N, cfg.num_v_heads, cfg.head_dim), dtype=_act(cfg), device=dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, cfg.num_v_heads, cfg.head_dim, cfg.head_dim),
                                  dtype=torch.float32, device=dev)
    if final_conv is None and return_final_conv:
        final_conv = torch.empty((B, cfg.conv_kernel - 1, cfg.conv_dim), dtype=_act(cfg),
                                 device=dev)
    o_raw = torch.empty((N, cfg.num_v_heads, cfg.head_dim), dtype=torch.float32,
                        device=dev) if return_o_raw else None
    need = prefill_workspace_size(cfg, B, N)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = lib().gdn_prefill(ctypes.byref(cfg._c()),
                           ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                           _ptr(qkv), _ptr(a), _ptr(b), _ptr(z), _ptr(cu_seqlens), B, N,
                           _ptr(initial_state), _ptr(initial_conv), _ptr(y), _ptr(final_state),
                           _ptr(final_conv), _ptr(o_raw), _ptr(workspace), workspace.numel(),
                           _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill")
    if check_status:
        dst, detail = prefill_status(workspace, stream)
        if dst != GDN_OK:
            raise GdnError(dst, f"gdn_prefill (device status, detail {detail:#010x})")
    out = {"y": y}
    if final_state is not None:
        out["final_state"] = final_state
    if final_conv is not None:
        out["final_conv"] = final_conv
    if o_raw is not None:
        out["o_raw"] = o_raw
    return out


def prefill_noalloc(cfg: Config, qkv, a, b, z, cu_seqlens, conv_w, A_log, dt_bias, norm_w, *,
                    y, initial_state=None, initial_conv=None, final_state=None, final_conv=None,
                    o_raw=None, stream=None) -> None:
    """gdn_prefill_noalloc: prefill into caller-provided outputs with the library's
    fixed internal scratch, for callers that cannot allocate device memory (a
    plugin whose host framework owns the GPU's memory, a loop that must never
    call cudaMalloc/cudaFree).  Nothing is allocated here or in the library.

    Calls on one device share the scratch: calls that overlap on the GPU race.
    The first call on a device looks up the scratch's address; make it before
    any stream capture.  Raises GdnError if the call needs more than
    NOALLOC_SCRATCH_BYTES of scratch (see prefill_workspace_size).  The device
    status of the call is read with prefill_noalloc_status()."""
    N = qkv.shape[0]
    B = cu_seqlens.shape[0] - 1
    st = lib().gdn_prefill_noalloc(ctypes.byref(cfg._c()),
                                   ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                                   _ptr(qkv), _ptr(a), _ptr(b), _ptr(z), _ptr(cu_seqlens), B, N,
                                   _ptr(initial_state), _ptr(initial_conv), _ptr(y),
                                   _ptr(final_state), _ptr(final_conv), _ptr(o_raw),
                                   _stream(stream))
    if st == GDN_ERR_WORKSPACE:
        raise GdnError(st, f"gdn_prefill_noalloc: needs {prefill_workspace_size(cfg, B, N)} bytes "
                           f"of scratch, more than the fixed {NOALLOC_SCRATCH_BYTES}")
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill_noalloc")


def decode(cfg: Config, qkv, a, b, z, state, conv_cache, conv_w, A_log, dt_bias, norm_w, *,
           y=None, stream=None):
    """One token per sequence; `state` and `conv_cache` are updated in place.  Returns y."""
    import torch
    B = qkv.shape[0]
    if y is None:
        y = torch.empty((B, cfg.num_v_heads, cfg.head_dim), dtype=_act(cfg), device=qkv.device)
    st = lib().gdn_decode(ctypes.byref(cfg._c()),
                          ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                          _ptr(qkv), _ptr(a), _ptr(b), _ptr(z), _ptr(state), _ptr(conv_cache), B,
                          _ptr(y), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode")
    return y


def _multi_y(cfg, qkv, y):
    import torch
    if y is None:
        B, k = qkv.shape[0], qkv.shape[1]
        y = torch.empty((B, k, cfg.num_v_heads, cfg.head_dim), dtype=_act(cfg), device=qkv.device)
    return y


def decode_multi(cfg: Config, qkv, a, b, z, state, conv_cache, conv_w, A_log, dt_bias, norm_w,
                 *, y=None, stream=None):
    """k tokens per sequence (qkv [B, k, conv_dim], a, b [B, k, H_v], z [B, k, H_v, d]);
    `state` and `conv_cache` advance by all k tokens in place.  Returns y [B, k, H_v, d]."""
    y = _multi_y(cfg, qkv, y)
    st = lib().gdn_decode_multi(ctypes.byref(cfg._c()),
                                ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                                _ptr(qkv), _ptr(a), _ptr(b), _ptr(z), _ptr(state),
                                _ptr(conv_cache), qkv.shape[0], qkv.shape[1], _ptr(y),
                                _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_multi")
    return y


def decode_verify(cfg: Config, qkv, a, b, z, state, conv_cache, conv_w, A_log, dt_bias, norm_w,
                  *, y=None, stream=None):
    """Outputs of k draft tokens per sequence; `state` and `conv_cache` are only read."""
    y = _multi_y(cfg, qkv, y)
    st = lib().gdn_decode_verify(ctypes.byref(cfg._c()),
                                 ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                                 _ptr(qkv), _ptr(a), _ptr(b), _ptr(z), _ptr(state),
                                 _ptr(conv_cache), qkv.shape[0], qkv.shape[1], _ptr(y),
                                 _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_verify")
    return y


def decode_commit(cfg: Config, qkv, a, b, state, conv_cache, accepted, conv_w, A_log, dt_bias,
                  norm_w, *, stream=None) -> None:
    """Advance `state` and `conv_cache` in place by the first accepted[n] tokens of each
    sequence (accepted: int32 tensor [B] on the device)."""
    st = lib().gdn_decode_commit(ctypes.byref(cfg._c()),
                                 ctypes.byref(_params(conv_w, A_log, dt_bias, norm_w)),
                                 _ptr(qkv), _ptr(a), _ptr(b), _ptr(state), _ptr(conv_cache),
                                 qkv.shape[0], qkv.shape[1], _ptr(accepted), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode_commit")


# ------------------------------------------------------------------ KDA


def kda_prefill_workspace_size(cfg: Config, batch: int, total_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    st = lib().gdn_kda_prefill_workspace_size(ctypes.byref(cfg._c()), batch, total_tokens,
                                              ctypes.byref(n))
    if st != GDN_OK:
        raise GdnError(st, "gdn_kda_prefill_workspace_size")
    return n.value


def kda_prefill(cfg: Config, qkv, zdec, b, gate, cu_seqlens, conv_w, A_log, norm_w, *,
                initial_state=None, initial_conv=None, return_final_state=False,
                return_final_conv=False, return_o_raw=False, y=None, final_state=None,
                final_conv=None, workspace=None, stream=None) -> dict:
    """Kimi Delta Attention prefill (gdn_kda_prefill): per-key-channel decay
    g = -5 sigmoid(exp(A_log) zdec), y = RMSNorm(o) * norm_w * sigmoid(gate)."""
    import torch
    N = qkv.shape[0]
    B = cu_seqlens.shape[0] - 1
    H, d, dev = cfg.num_v_heads, cfg.head_dim, qkv.device
    if y is None:
        y = torch.empty((N, H, d), dtype=_act(cfg), device=dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    if final_conv is None and return_final_conv:
        final_conv = torch.empty((B, cfg.conv_kernel - 1, cfg.conv_dim), dtype=_act(cfg), device=dev)
    o_raw = torch.empty((N, H, d), dtype=torch.float32, device=dev) if return_o_raw else None
    if workspace is None:
        workspace = torch.empty(max(kda_prefill_workspace_size(cfg, B, N), 1), dtype=torch.uint8,
                                device=dev)
    par = _KdaParams(_ptr(conv_w), _ptr(A_log), _ptr(norm_w))
    st = lib().gdn_kda_prefill(ctypes.byref(cfg._c()), ctypes.byref(par), _ptr(qkv), _ptr(zdec),
                               _ptr(b), _ptr(gate), _ptr(cu_seqlens), B, N, _ptr(initial_state),
                               _ptr(initial_conv), _ptr(y), _ptr(final_state), _ptr(final_conv),
                               _ptr(o_raw), _ptr(workspace), workspace.numel(), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_kda_prefill")
    out = {"y": y}
    if final_state is not None:
        out["final_state"] = final_state
    if final_conv is not None:
        out["final_conv"] = final_conv
    if o_raw is not None:
        out["o_raw"] = o_raw
    return out


def kda_decode(cfg: Config, qkv, zdec, b, gate, state, conv_cache, conv_w, A_log, norm_w, *,
               y=None, stream=None):
    """One KDA token per sequence; `state` and `conv_cache` are updated in place.  Returns y."""
    import torch
    B = qkv.shape[0]
    if y is None:
        y = torch.empty((B, cfg.num_v_heads, cfg.head_dim), dtype=_act(cfg), device=qkv.device)
    par = _KdaParams(_ptr(conv_w), _ptr(A_log), _ptr(norm_w))
    st = lib().gdn_kda_decode(ctypes.byref(cfg._c()), ctypes.byref(par), _ptr(qkv), _ptr(zdec),
                              _ptr(b), _ptr(gate), _ptr(state), _ptr(conv_cache), B, _ptr(y),
                              _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_kda_decode")
    return y
