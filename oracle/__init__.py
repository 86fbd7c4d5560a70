"""CPU fp64 oracle of the MoE expert layer -- TEST INFRASTRUCTURE ONLY (tests, smoke, bench baseline)."""
