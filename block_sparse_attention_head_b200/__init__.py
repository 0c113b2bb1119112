"""B200-native InstaGen group-shared importance-sampled permuted block-sparse attention."""
