"""B200-native MoE expert-parallel dispatch and combine (logical EP ranks on one GPU)."""
