"""CPU oracle of the token-choice MoE layer — test infrastructure only.

Imported by tests/, by __graft_entry__.smoke() and by bench.py's CPU
baseline; never by the library package.
"""
