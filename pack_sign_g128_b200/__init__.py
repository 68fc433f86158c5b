"""pack_sign_g128_b200: 1-bit group-128 matrix products on B200 (sm_100a)."""
