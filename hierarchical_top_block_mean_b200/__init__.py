"""B200-native PISA hot path (pyramid top-K block selection + block-sparse attention)."""
