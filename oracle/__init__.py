"""CPU oracle package -- TEST INFRASTRUCTURE (see oracle.py for the rules)."""
