"""B200-native FP8 W8A8 linear layers (binding filled in below)."""
