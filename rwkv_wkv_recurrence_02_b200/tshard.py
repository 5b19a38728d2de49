"""One long sequence split along T across ranks (one GPU per rank).

The skill page "rwkv-architecture" (agnxi.com) streams a million-token
document through chunks with the state carried from one to the next ("Process
million-token sequences").  Carried one chunk after another, the chunks run
one at a time.  Split across GPUs, every rank holds one consecutive chunk of
the sequence, and the only thing a chunk needs from the ones before it is the
state they leave behind.  A chunk's state from the empty state (its summary,
12 bytes per lane) folds associatively with the summaries before it (the scan
of "並列学習の定式化" in the article "RWKVアーキテクチャ徹底解説"), so one
exchange suffices:

  1. summary   every rank: wkv_state of its chunk from the empty state
               (reads k, v once);
  2. exchange  all-gather of the chunk lengths and the summaries
               (3 * B * C float32 per rank; NCCL over NVLink with the nccl
               backend);
  3. fold      wkv_state_combine of the summaries of ranks 0..rank-1 onto the
               sequence's initial state: the state entering this rank's chunk;
  4. forward   wkv_forward of this rank's chunk from that state.

Every rank takes the same collective steps in the same order.  Ranks hold
their chunks in rank order along T; chunk lengths may differ (0 included).
The traffic per rank is one extra read of k and v over a plain forward.

The arithmetic of steps 1, 3 and 4 is the CUDA library's (``ops`` defaults
to it); the argument exists so the exchange can be checked with ranks on CPU
against an independent implementation of the same three steps.
"""
import torch
import torch.distributed as dist

from . import wkv_forward, wkv_state, wkv_state_combine


class CudaOps:
    """Steps 1, 3 and 4 on the GPU through the C ABI."""

    def __init__(self, workspace=None, use_workspace=True):
        self.workspace = workspace
        self.use_workspace = use_workspace

    def state(self, w, k, v):
        return wkv_state(w, k, v, workspace=self.workspace, use_workspace=self.use_workspace)

    def combine(self, w, lens, states, state_in):
        return wkv_state_combine(w, lens, states, state_in)

    def forward(self, w, u, k, v, r, state_in, y):
        return wkv_forward(w, u, k, v, r, state_in, y=y, workspace=self.workspace,
                           use_workspace=self.use_workspace)


def forward_tsharded(w, u, k, v, r=None, state_in=None, *, y=None, group=None, ops=None):
    """Parallel mode over one sequence split along T across the ranks of
    `group`.  k, v, r: this rank's chunk (B, T_rank, C); w, u: (C,);
    state_in: the state entering the whole sequence (3, B, C), the same on
    every rank, or None for the empty state.  Returns (y, state_out): this
    chunk's outputs and the state after its last token (on the last rank, the
    state after the whole sequence)."""
    ops = CudaOps() if ops is None else ops
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, T, C = k.shape
    summary = ops.state(w, k, v).contiguous()
    # every rank's chunk length and summary, in rank order
    dev = summary.device
    lens_t = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(world)]
    dist.all_gather(lens_t, torch.tensor([T], dtype=torch.int64, device=dev), group=group)
    summaries = [torch.empty_like(summary) for _ in range(world)]
    dist.all_gather(summaries, summary, group=group)
    lens = [int(t.item()) for t in lens_t]
    if rank > 0:
        entering = ops.combine(w, lens[:rank], torch.stack(summaries[:rank]).contiguous(), state_in)
    else:
        entering = state_in
    return ops.forward(w, u, k, v, r, entering, y)
