"""B200-native DuoAttention hybrid-GQA attention (placeholder until the binding lands)."""
