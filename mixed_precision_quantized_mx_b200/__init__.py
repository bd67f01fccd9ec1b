"""B200-native MixLLM mixed-precision quantized linear layer (W4.4A8)."""
