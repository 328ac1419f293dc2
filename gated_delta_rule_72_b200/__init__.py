"""B200-native gated delta-net scan (causal, bidirectional, streaming step)."""
