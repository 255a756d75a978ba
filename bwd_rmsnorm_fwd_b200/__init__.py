"""B200-native training RMSNorm (forward, backward, residual form) behind a C-ABI library."""
