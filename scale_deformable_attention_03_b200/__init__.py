"""B200-native multi-scale deformable attention (placeholder; binding below)."""
