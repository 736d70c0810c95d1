"""B200-native (sm_100a) top-p block-sparse self-attention for video DiTs."""
