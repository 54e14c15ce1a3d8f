"""B200-native CGTP convolution (placeholder; the binding is added with the library)."""
