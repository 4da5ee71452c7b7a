"""B200-native QoQ W4A8 linear layer: Y = diag(s_x) (X8 W8hat^T) diag(s_c)."""
