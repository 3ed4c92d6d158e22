"""B200-native batch-1 MXFP4 MoE decode step (placeholder; the binding lands with the C-ABI library)."""
