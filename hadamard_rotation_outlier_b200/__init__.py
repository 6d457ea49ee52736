"""B200-native fused Hadamard rotate + quantize (placeholder; binding added next)."""
