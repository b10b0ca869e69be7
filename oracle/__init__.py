"""Plain CPU oracle of the TurboQuant quantizer (test infrastructure only:
tests/, the smoke check and bench.py's CPU-baseline leg)."""
