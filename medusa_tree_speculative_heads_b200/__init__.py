"""B200-native Medusa speculative decode step (binding package)."""
