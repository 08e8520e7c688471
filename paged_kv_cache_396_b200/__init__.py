"""B200-native paged decode attention library (Python side of the C ABI)."""
