"""CPU oracle for the stabilised BF16 FlashAttention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers or constant tables) and imports
neither torch nor the product package: NumPy float64 only.

Sources it restates (Qiu & Yao, "Why Low-Precision Transformer Training
Fails: An Analysis on Flash Attention", arXiv 2510.04212, as summarised by the
web pages "itsolotime.com/archives/23922" (page 1), "91haoming.cn ...
show-608006" (page 2) and their Thai translation (page 4)):

* ``bf16``      -- BF16 round-to-nearest-even emulation and the worked BF16
                   addition of page 2, section 4 ("the physical mechanism").
* ``attention`` -- safe-softmax attention forward (page 1, "mechanism two":
                   P_bar = exp(S - m), P = P_bar / rowsum, O = P V), the
                   stabilised shift rule (page 1, "minimal fix" pseudocode),
                   and the FlashAttention backward with delta = rowsum(dO o O)
                   (page 2, section 3).

Every function below is pinned by ``tests/test_oracle_*.py`` against values
that do not come from the oracle itself (closed forms, brute force, finite
differences, an independent library, the pages' worked example).
"""

from . import bf16, attention  # noqa: F401
