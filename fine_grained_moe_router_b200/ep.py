"""Expert-parallel forward of one fine-grained MoE layer across ranks (one GPU each).

"Kimi K3 fine-grained MoE under high concurrency", section "物理通信拓扑": each
token's copies travel to the ranks that own their experts (dispatch
All-to-All), the experts run there, and their outputs travel back (combine
All-to-All) to be weighted and summed with the shared expert's output; "MoE
architecture in production" §3.2 places the experts on different GPUs and
exchanges the tokens with NCCL All-to-All.

Rank r of G owns the experts [r*E/G, (r+1)*E/G) (E divisible by G) and holds
the gate, the shared expert and its own experts' weights. A forward of the
rank's T local tokens:

1. gate logits, top-K and renormalised weights (moe_router_topk), and the
   dispatch of the T*K copies over all E experts (moe_dispatch): sorted by
   expert, the copies are contiguous by owner rank;
2. the per-expert counts travel to the owners (All-to-All of [G, E/G] ints);
3. the dispatched rows x[perm / K] (moe_gather_rows) travel to the owners
   (All-to-All with the counts as split sizes), each rank into its own
   receive buffer;
4. the owner orders the received rows expert by expert (moe_ep_local_order)
   and runs its experts over them (moe_grouped_ffn, fp32 outputs);
5. the outputs go back to receive order (moe_gather_rows) and to their
   sources (All-to-All with the splits swapped), arriving in the source's
   dispatch order;
6. the source combines (moe_combine): y[t] = sum_k w[t,k] Yr[inv[t,k]] +
   S[t], with S[t] the shared expert's output on its own tokens, computed
   while the dispatched rows are in flight (step 3 runs asynchronously: the
   exchange overlaps that compute, the "communication masking" of the Kimi
   K3 page's section "工业级细粒度 MoE 路由与通信掩盖实战").

Every step of the arithmetic runs in libmoe's kernels through the C ABI;
torch.distributed carries the exchanges (NCCL over NVLink on GPUs: every
transfer lands in the receiving rank's own memory, and no kernel reads a
peer's memory). The split sizes of the row exchanges are read back to the
host once per forward. `ops` defaults to the CUDA library; another object with
the same methods can stand in for it where no GPU is present (tests run the
exchange logic on CPU ranks that way).
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


class CudaOps:
    """The compute steps of an expert-parallel forward, in libmoe's kernels."""

    def __init__(self):
        from . import _binding as B
        self.B = B
        self._ws = {}

    def _workspace(self, desc, device):
        n = self.B.moe_workspace_size(desc)
        ws = self._ws.get(device)
        if ws is None or ws.numel() < n:
            ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=device)
            self._ws[device] = ws
        return ws

    def _desc(self, T, H, E, K, D, Ds, dtype, cf):
        return self.B.make_desc(T, H, E, K, D, Ds, self.B.dtype_code(dtype), cf)

    def route(self, x, w_router, bias, K, cf):
        """(logits [T, E] fp32, topk_idx [T, K] int32, topk_w [T, K] fp32)."""
        T, H = x.shape
        E = w_router.shape[0]
        d = self._desc(T, H, E, K, 128, 0, x.dtype, cf)
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
        idx = torch.empty((T, K), dtype=torch.int32, device=x.device)
        w = torch.empty((T, K), dtype=torch.float32, device=x.device)
        self.B.moe_router_topk(d, x, w_router, bias, logits, idx, w, self._workspace(d, x.device))
        return logits, idx, w

    def dispatch(self, idx, E):
        """(counts [E], offsets [E+1], perm [T*K], inv [T*K]), int32."""
        T, K = idx.shape
        dev = idx.device
        d = self.B.make_desc(T, 128, E, K, 128, 0, self.B.MOE_BF16)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * K, dtype=torch.int32, device=dev)
        inv = torch.empty(T * K, dtype=torch.int32, device=dev)
        self.B.moe_dispatch(d, idx, counts, offsets, perm, inv, self._workspace(d, dev))
        return counts, offsets, perm, inv

    def gather_rows(self, src, idx, divisor):
        dst = torch.empty((idx.numel(), src.shape[1]), dtype=src.dtype, device=src.device)
        if idx.numel():
            self.B.moe_gather_rows(src, idx, divisor, dst)
        return dst

    def local_order(self, recv_counts):
        """(offsets [El+1], perm [R], inv [R]) of the received rows."""
        G, El = recv_counts.shape
        R = int(recv_counts.sum().item())
        dev = recv_counts.device
        offsets = torch.empty(El + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(R, dtype=torch.int32, device=dev)
        inv = torch.empty(R, dtype=torch.int32, device=dev)
        self.B.moe_ep_local_order(recv_counts.contiguous(), offsets, perm, inv)
        return offsets, perm, inv

    def experts(self, rows, perm, offsets, w1, w2):
        """y[j] = FFN_e(rows[perm[j]]) for j in expert e's segment (fp32 [R, H])."""
        R, H = rows.shape
        El, D, _ = w1.shape
        y = torch.empty((R, H), dtype=torch.float32, device=rows.device)
        if R == 0:
            return y
        d = self._desc(R, H, El, 1, D, 0, rows.dtype, (5, 4))
        self.B.moe_grouped_ffn(d, rows, perm, offsets, w1, w2, None, None, y, None,
                               self._workspace(d, rows.device))
        return y

    def combine(self, y_rows, topk_w, inv, y_shared, out_dtype):
        T, K = topk_w.shape
        H = y_rows.shape[1]
        y = torch.empty((T, H), dtype=out_dtype, device=y_rows.device)
        d = self._desc(T, H, max(K, 1), K, 128, 0, out_dtype, (5, 4))
        self.B.moe_combine(d, y_rows, topk_w, inv, y_shared, y)
        return y


class ExpertParallelMoE:
    """One MoE layer whose routed experts are spread over the ranks of `group`.

    w_router [E, H], w1_local [E/G, D, H], w2_local [E/G, H, D] (this rank's
    experts, in order), optional shared expert ws1 [Ds, H], ws2 [H, Ds] and
    fp32 expert bias [E]; every rank passes the same gate, bias and shared
    expert."""

    def __init__(self, w_router, w1_local, w2_local, top_k: int, ws1=None, ws2=None, bias=None,
                 group=None, ops=None, capacity_factor=(5, 4)):
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.H = w_router.shape
        if self.E % self.G:
            raise ValueError("the experts must split evenly over the ranks")
        self.El = self.E // self.G
        if w1_local.shape[0] != self.El or w2_local.shape[0] != self.El:
            raise ValueError("w1_local / w2_local must hold this rank's E/G experts")
        self.K = int(top_k)
        self.w_router, self.w1, self.w2 = w_router, w1_local, w2_local
        self.ws1, self.ws2, self.bias = ws1, ws2, bias
        self.cf = capacity_factor
        self.ops = ops if ops is not None else CudaOps()

    def forward(self, x: torch.Tensor, routing: Optional[dict] = None) -> torch.Tensor:
        """y = MoE(x) for this rank's tokens x [T, H]; `routing` (a dict) receives
        logits, topk_idx, topk_w, counts and recv_counts when given."""
        ops, G, El, K = self.ops, self.G, self.El, self.K
        logits, idx, w = ops.route(x, self.w_router, self.bias, K, self.cf)
        counts, offsets, perm, inv = ops.dispatch(idx, self.E)
        # 2. per-expert counts to the owners: row g of send_counts = rank g's experts
        send_counts = counts.reshape(G, El).contiguous()
        recv_counts = torch.empty_like(send_counts)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        send_splits = send_counts.sum(dim=1).tolist()
        recv_splits = recv_counts.sum(dim=1).tolist()
        # 3. the dispatched rows to the owners, in flight while the shared
        #    expert runs on this rank's tokens
        send_rows = ops.gather_rows(x, perm, K)
        recv_rows = torch.empty((sum(recv_splits), self.H), dtype=x.dtype, device=x.device)
        exchange = dist.all_to_all_single(recv_rows, send_rows, output_split_sizes=recv_splits,
                                          input_split_sizes=send_splits, group=self.group,
                                          async_op=True)
        y_shared = None
        if self.ws1 is not None:
            T = x.shape[0]
            tok = torch.arange(T, dtype=torch.int32, device=x.device)
            one = torch.tensor([0, T], dtype=torch.int32, device=x.device)
            y_shared = ops.experts(x, tok, one, self.ws1.unsqueeze(0), self.ws2.unsqueeze(0))
        exchange.wait()
        # 4. this rank's experts over the received rows, expert by expert
        loc_off, loc_perm, loc_inv = ops.local_order(recv_counts)
        y_local = ops.experts(recv_rows, loc_perm, loc_off, self.w1, self.w2)
        # 5. back to receive order, then to the sources (their dispatch order)
        y_back = ops.gather_rows(y_local, loc_inv, 1)
        y_rows = torch.empty((perm.numel(), self.H), dtype=y_back.dtype, device=x.device)
        dist.all_to_all_single(y_rows, y_back, output_split_sizes=send_splits,
                               input_split_sizes=recv_splits, group=self.group)
        # 6. combine with the shared expert's output
        y = ops.combine(y_rows, w, inv, y_shared, x.dtype)
        if routing is not None:
            routing.update(logits=logits, topk_idx=idx, topk_w=w, counts=counts,
                           recv_counts=recv_counts)
        return y

    __call__ = forward
