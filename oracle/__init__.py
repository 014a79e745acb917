"""CPU oracle of the PIVOT indexer: test infrastructure only (see oracle.py)."""
