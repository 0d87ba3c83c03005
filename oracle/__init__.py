"""Plain float64 CPU oracle for Sliding Tile Attention (STA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arms of ``bench.py`` may import or run it.  It shares no code with the CUDA
library in ``block_sparse_local_b200/``; the two meet only through the seeded
input generator ``block_sparse_local_b200/workloads.py``, which holds none of
the method's arithmetic.

Source of the method: the README "Sliding Tile Atteniton Kernel" of the
FastVideo STA kernel (sta_kernel/thunderkitten), sections "Usage",
"How Does STA Work?" and "Why is STA Fast?".  The 1-D sliding-window
comparison follows the sliding-window-attention search-result page
(Mistral 7B sliding window over 4096 previous states, GQA; causal band
decomposed into invisible, upper- and lower-triangular blocks).

Modules:
  sta_oracle    - attention itself (dense-mask form A and row-gather form B)
  tiles_oracle  - per-query-tile KV tile lists (brute-force box test)
  perm_oracle   - raster <-> tile token permutation (index formula)
  swa_oracle    - token-level causal sliding-window attention with GQA

Every function is pinned by a ``-m "not gpu"`` test in tests/test_oracle*.py
except where its docstring says "parity unpinned".
"""
