"""CPU oracle for the SAS gated block-sparse attention path (test infrastructure only)."""
