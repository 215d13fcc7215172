"""Gated bidirectional ReLU linear attention on B200 (sm_100a)."""
