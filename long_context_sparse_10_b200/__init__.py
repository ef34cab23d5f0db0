"""B200-native CSA / HCA hybrid attention (placeholder; binding added with the library)."""
