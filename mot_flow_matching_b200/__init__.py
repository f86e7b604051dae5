"""B200-native gen-tower attention layer (MoT flow-matching denoise step)."""
