"""CPU oracle for decode-time QSA (test infrastructure only; see qsa_ref)."""
