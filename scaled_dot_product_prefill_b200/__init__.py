"""B200-native exact scaled-dot-product attention: tiled prefill and paged decode."""
