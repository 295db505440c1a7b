"""The oracle: a plain CPU statement of paged decode attention (test infrastructure only)."""
