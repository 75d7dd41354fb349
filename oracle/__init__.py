"""CPU oracle of the LLM.int8() linear layer (test infrastructure only; see oracle.py)."""
