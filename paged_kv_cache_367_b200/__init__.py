"""B200-native paged KV append and PagedAttention decode."""
