"""Sparse index attention on B200: indexer score -> Top-K -> sparse MLA over a paged latent cache."""
