"""B200-native forward pass of a DeepSeek-V3-style MoE feed-forward layer."""
