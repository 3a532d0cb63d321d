"""Block-sparse 3D spatio-temporal attention for video-DiT tokens on B200 (sm_100a)."""
