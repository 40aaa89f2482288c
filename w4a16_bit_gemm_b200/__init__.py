"""B200-native group-wise RTN weight quantization and W4A16 linear layers."""
