"""fp64 CPU oracle for paged latent attention: test infrastructure only (see mla_oracle)."""
