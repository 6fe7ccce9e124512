"""fp64 CPU oracle for exact attention (test infrastructure; see attention.py)."""

from .attention import attention_backward_ref, attention_bruteforce, attention_ref, visibility
from .philox import dropout_keep, dropout_threshold, philox4x32, philox4x64_py

__all__ = ["attention_ref", "attention_bruteforce", "attention_backward_ref", "visibility", "dropout_keep",
           "dropout_threshold", "philox4x32", "philox4x64_py"]
