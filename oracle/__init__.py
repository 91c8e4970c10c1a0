"""Float64 CPU oracle of the latent KV cache (test infrastructure only)."""
