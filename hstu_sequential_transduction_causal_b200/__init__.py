"""B200-native HSTU layer (pointwise-attention sequential transduction) behind a C ABI."""
