"""Latent mixture-of-experts FFN block for NVIDIA B200 (sm_100a)."""
