"""B200-native chunked Gated DeltaNet (GDN) scan."""
