"""CPU oracle for the Video DeltaNet hybrid attention layer (float64, numpy).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code, table or helper with the CUDA library; both sides receive the
same seeded input arrays and nothing else.

Every function here is the plain definition of one step, written from the
pages' description of the method:

* ``vda``          -- Video Delta Attention (frame-level delta rule, closed
                      form S_t = (S_bar_t + B_t)(I + A_t)^-1, run forward and
                      backward over the latent frames).  Source: "Video
                      DeltaNet" article on 10100.com, section 方法概述 item 2
                      (frame-level delta rule), figure caption under
                      效率阶梯 (forward and backward scans).
* ``window_attn``  -- sliding-window Softmax over 5-frame chunks (+-1 chunk)
                      with first/last-frame anchors.  Source: same article,
                      方法概述 item 1 (Sliding-Window Softmax + Boundary
                      Anchors).
* ``fuse``         -- branch calibration: content-dependent sigmoid gate on
                      the Softmax branch, RMSNorm then sigmoid output gate on
                      the linear branch, separate output projections, summed.
                      Source: same article, 方法概述 item 3.

* ``vda_backward`` -- gradients of the VDA output with respect to q, k, v,
                      beta and alpha (adjoint scans), for training the branch.
* ``mxfp8``        -- MXFP8 quantization (E4M3 elements, UE8M0 block scales)
                      and the fuse with MXFP8 projections.

The readings taken where the pages are silent are stated in each module's
docstring.  Parity status of every function is pinned by the
``-m "not gpu"`` tests in ``tests/test_oracle_pins.py``; none is unpinned.
"""

from .vda import (vda_prep, vda_frame_state, vda_scan, vda_readout, vda,
                  transition_matrix)
from .window_attn import (frame_visible, visible_key_frames, window_attn,
                          window_attn_rows, mask_pair_count)
from .fuse import sigmoid, rmsnorm_heads, fuse_gates, hybrid_fuse, hybrid_fuse_rows
from .vda_backward import vda_backward
from . import mxfp8

__all__ = [
    "vda_prep", "vda_frame_state", "vda_scan", "vda_readout", "vda",
    "transition_matrix",
    "frame_visible", "visible_key_frames", "window_attn", "window_attn_rows",
    "mask_pair_count",
    "sigmoid", "rmsnorm_heads", "fuse_gates", "hybrid_fuse", "hybrid_fuse_rows",
    "vda_backward", "mxfp8",
]
