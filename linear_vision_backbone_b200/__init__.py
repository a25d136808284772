"""B200-native Key-only gated linear attention (GTR token mixer)."""
