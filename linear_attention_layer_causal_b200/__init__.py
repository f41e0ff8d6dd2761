"""B200 (sm_100a) Gated DeltaNet token mixer: placeholder until the binding lands."""
