"""verify_step_lm_b200: B200-native speculative-decoding verify step."""
