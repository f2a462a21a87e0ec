"""CPU oracle for radial block-sparse attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything here. The CUDA library in
``block_sparse_attention_radial_b200`` shares no code with this package and
never imports it.

Everything is plain NumPy in float64. Pages cited (tag: page title, site):

* [RA-skill]  "Radial Attention: O(nlog n) Sparse Attention with Energy Decay
  for Long Video Generation" skill page (skillsmp.com, radial-attention-video):
  Step 1 (mask), Step 2 (RadialAttention module), hyper-parameter table.
* [RA-summary] the same paper's summary page (slashpage.com), "Outline".
* [RA-blog]   "Radial Attention: A Breakthrough in Efficient Long Video
  Generation" (thismoment.ai), "How Radial Attention Works".
* [vDiT-skill] "Sparse-vDiT: Unleashing the Power of Sparse Attention to
  Accelerate Video Diffusion Transformers" skill page (skillsmp.com),
  "Sparse attention patterns".
* [CA-abstract] Compact Attention abstract (zhuanzhiai.com).

Modules:

* ``radial_mask``: the token-level radial rule and two independent block-list
  constructions (brute force over the token mask; per-token key intervals);
  the joint text + video lists (text tokens appended, attended globally).
* ``attention``: masked softmax attention over block lists, in float64.
* ``attention_backward``: its gradients (dQ, dK, dV), in float64.
* ``module``: the RadialAttention module forward (projections, head split,
  attention, head merge, output projection), in float64.
* ``tile_patterns``: per-head tile patterns (diagonal and multi-diagonal
  bands, vertical stripes, dual windows) expanded into block lists.
* ``varlen``: variable-length batches (items with their own lists,
  concatenated; attention and its gradients item by item).
"""

from .radial_mask import (  # noqa: F401
    band_index,
    r_star,
    window_width,
    keep_frame,
    window_start,
    radial_token_mask,
    block_lists_from_token_mask,
    radial_block_lists_bruteforce,
    radial_block_lists_intervals,
    radial_block_lists,
    joint_token_mask,
    joint_block_lists_bruteforce,
    joint_block_lists,
)
from .attention import (  # noqa: F401
    expand_row_mask,
    masked_attention_rows,
    masked_attention_fp64,
    bf16_round,
)
from .attention_backward import (  # noqa: F401
    masked_attention_backward_fp64,
    masked_attention_dq_rows,
    masked_attention_dkdv_keys,
)
from .tile_patterns import (  # noqa: F401
    tile_pattern_mask,
    tile_pattern_lists,
)
from .varlen import (  # noqa: F401
    varlen_block_lists,
    split_item_lists,
    varlen_masked_attention_fp64,
    varlen_masked_attention_backward_fp64,
)
from .module import (  # noqa: F401
    radial_attention_module_fp64,
    radial_attention_module_backward_fp64,
    radial_attention_module_rows,
)
