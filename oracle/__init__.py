"""CPU float64 oracle for calibrated block-sparse attention (CalibAtt).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only the test-suite, the smoke check and the benchmark's CPU
baseline leg use it.  It shares no code, constants or helpers with the CUDA
library; both sides only receive the same seeded inputs.

Source: "Accelerating Text-to-Video Generation with Calibrated Sparse
Attention" (Yehezkel, Yadin, Elata, Ostrovsky-Berman, Kawar; arXiv 2603.05503),
as reproduced on its paper page: the Abstract, Figures 2-5 and Table S3.

Functions (each is the plain definition or the plain step sequence; no
blocking, fusion or reordering beyond what the definition states):

* ``masked_attention``  -- softmax attention restricted to kept key blocks
  (Abstract: "compute the selected ... connections densely, and skip the
  unselected ones"; Figure 5(b) top).
* ``block_energy``      -- post-softmax attention mass per (query block, key
  block) (Figure 2 "block-level" post-softmax maps; Table S5 "block
  energies").
* ``select_topk`` / ``select_energy`` -- per-query-block thresholding of the
  top key blocks (Figure 5(a); Figure S8 energy threshold).
* ``vote``               -- agreement voting across calibration inputs
  (Figure 3(b) keep frequency; Figure 7 agreement threshold rho).
* ``timestep_clusters`` / ``share_masks`` -- timestep sharing of calibrated
  masks (Figure S11 skipped-block IoU across timesteps; Table S3 clusters of
  pair-wise IoU >= tau).
* ``interval_counts`` / ``merge_masks`` / ``skiplist_bytes`` -- the pages'
  interval skip-list storage (Figure S9, Figure S10, Table S3).
* ``anchor_rows`` / ``anchor_attention`` -- spatial repetition: attention of
  k anchor rows per frame broadcast to the other rows (Figure 4, Figure 5(b)
  bottom, Table S4).
* ``spatial_similarity`` / ``repetition_flags`` -- the per-head spatial
  similarity score and the repetition dictionary (Figure 5(a), Figure 6,
  Figure S13; the score's definition is this build's reading).
* ``compile_blocklist`` / ``expand_blocklist`` -- compile masks into per-row
  kept-block lists with translation-relative row-pattern dedup (Abstract:
  "compiles these patterns into optimized attention operations for each
  layer, head, and diffusion timestep"; Figure 4(b): the pattern repeats
  across spatial rows).

Parity status: every function here is pinned by tests under ``tests/`` that
do not re-type its formula (textbook SDPA, brute-force loops, closed forms,
invariants).  The energy-threshold selection is pinned by brute force, but the
pages print no epsilon values, so its *schedule* is unpinned (parity unpinned
for epsilon values, not for the selection rule).
"""

from .attention import masked_attention, masked_attention_rows
from .calibration import block_energy, block_energy_row, select_topk, select_energy, topk_count, vote, min_votes_for
from .compile import compile_blocklist, expand_blocklist
from .sharing import skipped_iou, timestep_similarity, timestep_clusters, share_masks
from .skiplist import interval_counts, merge_row, merge_masks, nearest_rank, skiplist_bytes
from .anchor import anchor_rows, anchor_attention, anchor_attention_tokens, spatial_similarity, repetition_flags

__all__ = [
    "masked_attention",
    "masked_attention_rows",
    "block_energy",
    "select_topk",
    "select_energy",
    "topk_count",
    "vote",
    "min_votes_for",
    "compile_blocklist",
    "expand_blocklist",
]
