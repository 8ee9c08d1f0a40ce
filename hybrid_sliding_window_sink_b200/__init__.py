"""Attention-sink softmax attention for hybrid SWA/GA decoders on B200 (sm_100a)."""
