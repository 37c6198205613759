"""B200-native Multi-Head Latent Attention decode (absorbed form, paged latent cache)."""
