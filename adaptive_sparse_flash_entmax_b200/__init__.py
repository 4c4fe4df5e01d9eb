"""B200-native fused alpha-entmax attention (AdaSplash-style), forward and backward."""
