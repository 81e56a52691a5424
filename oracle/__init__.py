"""fp64 CPU oracle for the VideoMLA latent-KV hot path (test infrastructure only)."""
