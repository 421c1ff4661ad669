"""B200-native Kalman Linear Attention filter scan (binding added with the CUDA library)."""
