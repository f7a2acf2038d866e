"""fp64 CPU oracle of the latent mixture-of-experts FFN block (test infrastructure only)."""
