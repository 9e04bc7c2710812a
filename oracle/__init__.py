"""CPU oracle for TurboQuant-prod KV-cache compression and compressed-KV decode.

TEST INFRASTRUCTURE ONLY.  This package is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by ``bench.py``'s CPU-baseline / reference
leg, and by nothing else.  The product (the CUDA library and its Python
binding) never imports, links or executes anything here, and nothing here
imports the product.  The only module both sides share is the seeded input
generator ``kv_cache_quantization_turboquantprod_b200.workloads``, which holds
none of the method's arithmetic.

Plain, slow, float64 NumPy written from the pages' statement of the method:

* ``codebook``  -- Lloyd-Max scalar codebook for the post-rotation coordinate
  law (Gaussian N(0, 1/d) reading).
* ``quant``     -- TurboQuant-prod key encoding (normalise, rotate, bucketize,
  residual, 1-bit QJL sketch, norms) and group quantization of values.
* ``layout``    -- the byte layout of the compressed cache, written from its
  prose specification (pack and unpack).
* ``attention`` -- the unbiased inner-product score, one-pass decode attention
  over the compressed cache, explicit dequantization, and the brute-force
  softmax over dequantized K/V.
* ``accounting`` -- storage bytes and compression ratios.

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against closed forms, textbook constants, the pages' printed numbers or
brute force (see tests/test_oracle_*.py).  No function is "parity unpinned".
"""

from . import accounting, attention, codebook, layout, quant  # noqa: F401
