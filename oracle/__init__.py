"""Test infrastructure only: the double-precision CPU oracle of the HGA hot path."""
