"""B200-native Kimi Delta Attention (KDA) operator: package root (filled in below)."""
