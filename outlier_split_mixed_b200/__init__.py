"""B200-native smoothed, outlier-split W4A4 linear layer (placeholder binding)."""
