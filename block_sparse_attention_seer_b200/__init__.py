"""B200-native gated block-sparse decode attention (SeerAttention-R hot path)."""
