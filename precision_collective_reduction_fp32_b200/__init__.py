"""B200-native emulated RCCLX collectives (DDA allreduce, FP8 low-precision collectives)."""
