"""Memory-efficient elementwise activations for B200 (placeholder; binding follows)."""
