"""Load-balanced MoE token dispatch and combine for B200 (sm_100a)."""
