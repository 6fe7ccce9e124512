"""fp64 CPU oracle for exact attention (test infrastructure; see attention.py)."""

from .attention import attention_backward_ref, attention_bruteforce, attention_ref, visibility

__all__ = ["attention_ref", "attention_bruteforce", "attention_backward_ref", "visibility"]
