"""A decode step captured into a CUDA graph.

One decode step is a short chain of launches: the cache append of the new
K/V rows, the decode kernel, and (when long contexts are split) the merge of
the partitions.  For small batches the launch overhead is comparable to the
work, so the chain is captured once and replayed ("大模型推理优化：KV Cache与
FlashAttention实战" §5.2 and "Flash Attention与Paged KV Cache优化大模型计算效率"
§4.1 capture the decode critical path in a CUDA graph).

The graph holds the device pointers of the tensors given here: between
replays the caller updates their *contents* in place (new q, new K/V rows and
slots, block tables, context lengths) and calls :meth:`replay`.  Shapes, and
therefore the split-KV plan, are fixed at capture time; context lengths may
change freely up to ``max_pages_per_seq * page_size``.
"""
from __future__ import annotations

import torch

from . import ops


class DecodeStepGraph:
    def __init__(self, q, k_pages, v_pages, block_tables, context_lens, scale, *, k_new=None, v_new=None,
                 slot_mapping=None, out=None, k_scales=None, v_scales=None, num_splits=0):
        B, Hq, D = q.shape
        P, ps, Hkv, _ = k_pages.shape
        self.out = torch.empty_like(q) if out is None else out
        need = ops.decode_workspace_size(B, Hq, Hkv, D, ps, block_tables.shape[1], k_pages.dtype, num_splits)
        self.workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        self._args = (q, k_pages, v_pages, block_tables, context_lens, scale)
        self._kw = dict(k_scales=k_scales, v_scales=v_scales, workspace=self.workspace, num_splits=num_splits)
        self._new = (k_new, v_new, slot_mapping) if k_new is not None else None
        # One eager run on a side stream does the per-device set-up (device symbol
        # lookup, kernel attributes) outside the capture.
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._step()

    def _step(self):
        if self._new is not None:
            k_new, v_new, slots = self._new
            ops.kv_cache_write(k_new, v_new, slots, self._args[1], self._args[2])
        ops.paged_attention_decode(*self._args, self.out, **self._kw)

    def replay(self):
        """Run the captured step on the current stream; returns the output tensor."""
        self.graph.replay()
        return self.out
