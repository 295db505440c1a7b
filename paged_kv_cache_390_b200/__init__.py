"""B200-native paged decode attention: a C-ABI CUDA library and its Python binding."""
