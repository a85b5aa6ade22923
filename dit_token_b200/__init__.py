"""Fused per-token operators of a packed audio-video DiT block for B200."""
