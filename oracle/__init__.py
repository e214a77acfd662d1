"""Plain float64 CPU oracle for exact long-context attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path (the
C-ABI library and its Python binding) never imports, links or runs anything
here, and this package imports nothing from the product path.

Modules:
  attention  exact attention rows, single-token decode, log-sum-exp merge
  fp8        E4M3 code table from the format definition
  intq       INT8 / INT4 KV codes (two's complement, low nibble first) to values
  stream     exact-cover check of a (query block, key chunk) task list
  paged      paged KV cache: gather mapped pages into the contiguous cache, then decode
"""
