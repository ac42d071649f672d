"""dit_block_pass_b200: B200-native (sm_100a) memory-bound operators of a dense
single-stream video+audio DiT block."""
