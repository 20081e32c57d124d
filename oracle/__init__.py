"""fp64 CPU oracle for paged KV-cache attention (test infrastructure only)."""
