"""B200-native top-k mixture-of-experts FFN layer (DiffusionGemma 26B-A4B shape)."""
