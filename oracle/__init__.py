"""CPU oracle (test infrastructure only): see ``oracle.moba_ref``."""
