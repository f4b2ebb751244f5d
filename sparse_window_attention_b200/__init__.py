"""BASA shifted-window sparse attention, forward hot path for B200 (sm_100a)."""
