"""B200-native Exact Flow Linear Attention (EFLA) forward pass."""
