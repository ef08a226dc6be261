"""Simple GLA mixer on B200 (placeholder until the binding lands)."""
