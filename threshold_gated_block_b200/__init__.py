"""B200-native BSFA (threshold-gated block-sparse flash attention) prefill forward."""
