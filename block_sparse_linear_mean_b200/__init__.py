"""B200-native hybrid block-sparse + linear attention (SLA / NABLA style)."""
