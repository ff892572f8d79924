"""TurboQuant KV-cache oracle (TEST INFRASTRUCTURE ONLY; see oracle.py)."""
