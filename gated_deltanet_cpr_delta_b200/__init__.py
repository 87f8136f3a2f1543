"""CPR Gated DeltaNet for B200 (sm_100a): C-ABI library + thin Python binding."""
