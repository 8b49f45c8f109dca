"""B200-native fused MoE expert layer: routed grouped GEMMs behind a C ABI."""
