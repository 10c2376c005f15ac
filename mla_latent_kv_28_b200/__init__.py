"""B200-native MLA absorbed-decode library: the Python side of the C ABI."""
