"""CAAT-Net partially synchronized row-parallel layer: B200-native C-ABI library."""
