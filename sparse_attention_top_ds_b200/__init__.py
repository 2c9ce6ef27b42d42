"""B200-native selection step of DeepSeek-style sparse attention (placeholder)."""
