"""Plain, slow, double-precision CPU oracle for the TurboQuant compressed-KV path.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check of the package entry
point and the CPU-baseline leg of the benchmark may import this package. The
product library (the CUDA kernels behind the C ABI) never calls it, and it
shares no code, headers, tables or constants with the product.

Every function follows the pages it cites in the order and notation they give:

* "turboquant_cutile" function list (codehub.bot page for DevTechJr/turboquant_cutile):
  the API statement - compress K (MSE + QJL), compress V (MSE only), the
  asymmetric estimator, the attention pipeline, decompression as
  "indices -> centroids -> un-rotate -> rescale", codebook as sorted float32
  centroids/boundaries.
* "TurboQuant explained: near-optimal KV cache compression ..." (Mobilint blog):
  the mathematics - the Walsh-Hadamard/Rademacher rotation HD, the Beta density
  of rotated coordinates, Lloyd-Max, the QJL estimator, the two-stage
  TurboQuant_prod quantizer and its bounds.
* "tq-kv" crate documentation (docs.rs): pre-rotated query and centroid-table
  scoring.

Modules:
  codebook   - rotated-coordinate densities and the Lloyd-Max codebook
  rotation   - Sylvester Walsh-Hadamard, HD and dense rotations
  quant      - per-vector norm, quantize/dequantize, TurboQuant_mse / _prod compression
  layout     - the packed page format (an encoding the pages leave open)
  attention  - estimator, decode attention over packed pages, exact attention

Parity status: every function here is pinned by tests/test_oracle_*.py against
values printed on the pages, closed forms, invariants, library routines or brute
force, except the items listed as "parity unpinned" in the module docstrings.
"""

from . import codebook, rotation, quant, layout, attention  # noqa: F401
