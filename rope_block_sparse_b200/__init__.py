"""B200-native attention core for H3-style video DiTs."""
