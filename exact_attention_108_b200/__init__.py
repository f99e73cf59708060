"""B200-native exact attention: Python binding over the C-ABI library ``libfattn.so``.

Importing the package loads nothing; the shared library is opened on first use
and a missing library is a hard error (there is no fallback path).
"""
