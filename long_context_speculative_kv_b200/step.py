"""One Windowed-MTP decode step issued through the library, in the order of the pages' cost
identity (Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery, Eq. 1):

    t_step = t_ctx_draft + gamma * t_fwd_draft + t_verify (+ acceptance)

  * t_ctx_draft: append the gamma + 1 committed tokens' draft K/V, then one draft attention call
    with n_q = gamma + 1 (worst case: every draft of the previous step accepted);
  * t_fwd_draft: append one draft K/V row, then one draft attention call with n_q = 1;
    in the windowed arm each of these pairs is one library call (draft_attn_window_append: the
    append happens inside the attention kernel);
  * t_verify:    one verify_attn call per target attention layer (n_q = gamma + 1, or the tree);
  * acceptance:  accept_greedy over the verify step's logits.

The windowed arm reads the draft KV from the compact ring (draft_attn_window); the native arm
reads the whole paged draft cache (draft_attn_full).  Only the draft terms differ.  The native
arm's own cache write of the new draft rows belongs to the model's KV store, not to this
attention path, and is not issued.

The class owns no arithmetic: it holds device buffers (filled by the caller's generator) and
issues library calls on the current stream, recording CUDA events between calls when asked.
"""
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

from . import api


@dataclass
class StepBuffers:
    # verify
    k_pools: List[torch.Tensor]
    v_pools: List[torch.Tensor]
    table_v: torch.Tensor
    kv_len_v: torch.Tensor
    q_verify: torch.Tensor              # [layers, B, n_q, Hq, D]
    tree_parent: Optional[torch.Tensor]
    logits: torch.Tensor                # [B, n_q, V]
    tokens: torch.Tensor                # [B, n_q]
    # draft (both arms share queries and new rows)
    q_ctx: torch.Tensor                 # [B, gamma + 1, Hq, D]
    q_fwd: torch.Tensor                 # [gamma, B, 1, Hq, D]
    k_ctx: torch.Tensor                 # [B, gamma + 1, Hkv, D]
    v_ctx: torch.Tensor
    k_fwd: torch.Tensor                 # [gamma, B, 1, Hkv, D]
    v_fwd: torch.Tensor
    # windowed arm
    ring_k: Optional[torch.Tensor] = None
    ring_v: Optional[torch.Tensor] = None
    ring_len: Optional[torch.Tensor] = None
    n_sink: int = 4
    window: int = 4092
    # native arm
    k_draft: Optional[torch.Tensor] = None
    v_draft: Optional[torch.Tensor] = None
    table_d: Optional[torch.Tensor] = None
    kv_len_ctx: Optional[torch.Tensor] = None
    kv_len_fwd: Optional[List[torch.Tensor]] = None
    sm_scale: float = 128 ** -0.5
    # fp8 (E4M3) KV: every K/V cache and new row holds codes, scaled by k_scale / v_scale
    kv8: bool = False
    k_scale: float = 1.0
    v_scale: float = 1.0
    # outputs / workspace
    ws: Optional[torch.Tensor] = None
    out: Dict[str, torch.Tensor] = field(default_factory=dict)


class CallLog:
    """Events between consecutive library calls of one step: call k runs between events k and
    k + 1 (calls are back to back on one stream)."""

    def __init__(self):
        self.labels: List[str] = []
        self.events: List[torch.cuda.Event] = []

    def mark(self, label: Optional[str]):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.events.append(e)
        if label is not None:
            self.labels.append(label)

    def durations_ms(self):
        return [(lab, self.events[i].elapsed_time(self.events[i + 1]))
                for i, lab in enumerate(self.labels)]


class DecodeStep:
    def __init__(self, bufs: StepBuffers, gamma: int):
        self.b = bufs
        self.gamma = gamma
        B, n_q, Hq, _ = bufs.q_verify.shape[1:]
        self.n_layers = bufs.q_verify.shape[0]
        self.n_q_verify = n_q
        b = bufs
        b.out["verify"] = torch.empty_like(bufs.q_verify[0])
        b.out["verify_lse"] = torch.empty(bufs.q_verify.shape[1:4], dtype=torch.float32,
                                          device=bufs.q_verify.device)
        b.out["ctx"] = torch.empty_like(bufs.q_ctx)
        b.out["ctx_lse"] = torch.empty(bufs.q_ctx.shape[:3], dtype=torch.float32, device=bufs.q_ctx.device)
        b.out["fwd"] = torch.empty_like(bufs.q_fwd[0])
        b.out["fwd_lse"] = torch.empty(bufs.q_fwd.shape[1:4], dtype=torch.float32, device=bufs.q_fwd.device)
        b.out["accepted"] = torch.empty(bufs.tokens.shape, dtype=torch.int32, device=bufs.tokens.device)
        b.out["n_accepted"] = torch.empty(bufs.tokens.shape[:1], dtype=torch.int32, device=bufs.tokens.device)
        if b.ws is None:
            Hkv = bufs.k_pools[0].shape[1]
            need = max(api.workspace_bytes(B, max(n_q, gamma + 1), Hq, Hkv),
                       api.workspace_bytes(B, 1, Hq, Hkv))
            b.ws = torch.zeros(need, dtype=torch.uint8, device=bufs.q_verify.device)

    # ----------------------------------------------------------------------------- phases
    def draft_windowed(self, log: Optional[CallLog] = None):
        b = self.b
        if log: log.mark("window_ctx")
        self._forward(b.q_ctx, b.k_ctx, b.v_ctx, b.out["ctx"], b.out["ctx_lse"])
        for j in range(self.gamma):
            if log: log.mark("window_fwd")
            self._forward(b.q_fwd[j], b.k_fwd[j], b.v_fwd[j], b.out["fwd"], b.out["fwd_lse"])

    def _forward(self, q, k_new, v_new, out, lse):
        """Ring append of the new rows and the windowed attention, one library call."""
        b = self.b
        if b.kv8:
            api.draft_attn_window_append_fp8(q, b.ring_k, b.ring_v, b.ring_len, k_new, v_new, b.n_sink,
                                             b.window, b.sm_scale, b.k_scale, b.v_scale, b.ws,
                                             out=out, lse=lse)
        else:
            api.draft_attn_window_append(q, b.ring_k, b.ring_v, b.ring_len, k_new, v_new, b.n_sink,
                                         b.window, b.sm_scale, b.ws, out=out, lse=lse)

    def _append(self, k_new, v_new):
        b = self.b
        if b.kv8:
            api.ring_kv_append_fp8(b.ring_k, b.ring_v, b.ring_len, k_new, v_new, b.n_sink)
        else:
            api.ring_kv_append(b.ring_k, b.ring_v, b.ring_len, k_new, v_new, b.n_sink)

    def _window(self, q, out, lse):
        b = self.b
        if b.kv8:
            api.draft_attn_window_fp8(q, b.ring_k, b.ring_v, b.ring_len, b.n_sink, b.window, b.sm_scale,
                                      b.k_scale, b.v_scale, b.ws, out=out, lse=lse)
        else:
            api.draft_attn_window(q, b.ring_k, b.ring_v, b.ring_len, b.n_sink, b.window, b.sm_scale,
                                  b.ws, out=out, lse=lse)

    def _full(self, q, kv_len, out, lse):
        b = self.b
        if b.kv8:
            api.draft_attn_full_fp8(q, b.k_draft, b.v_draft, b.table_d, kv_len, b.sm_scale, b.k_scale,
                                    b.v_scale, b.ws, out=out, lse=lse)
        else:
            api.draft_attn_full(q, b.k_draft, b.v_draft, b.table_d, kv_len, b.sm_scale, b.ws, out=out, lse=lse)

    def draft_native(self, log: Optional[CallLog] = None):
        b = self.b
        if log: log.mark("full_ctx")
        self._full(b.q_ctx, b.kv_len_ctx, b.out["ctx"], b.out["ctx_lse"])
        for j in range(self.gamma):
            if log: log.mark("full_fwd")
            self._full(b.q_fwd[j], b.kv_len_fwd[j], b.out["fwd"], b.out["fwd_lse"])

    def verify(self, log: Optional[CallLog] = None):
        b = self.b
        for layer in range(self.n_layers):
            if log: log.mark("verify")
            if b.kv8:
                api.verify_attn_fp8(b.q_verify[layer], b.k_pools[layer], b.v_pools[layer], b.table_v,
                                    b.kv_len_v, b.sm_scale, b.k_scale, b.v_scale, b.ws,
                                    tree_parent=b.tree_parent, out=b.out["verify"], lse=b.out["verify_lse"])
            else:
                api.verify_attn(b.q_verify[layer], b.k_pools[layer], b.v_pools[layer], b.table_v,
                                b.kv_len_v, b.sm_scale, b.ws, tree_parent=b.tree_parent,
                                out=b.out["verify"], lse=b.out["verify_lse"])

    def accept(self, log: Optional[CallLog] = None):
        b = self.b
        if log: log.mark("accept")
        api.accept_greedy(b.logits, b.tokens, b.tree_parent, accepted=b.out["accepted"],
                          n_accepted=b.out["n_accepted"])

    def run(self, arm: str, log: Optional[CallLog] = None):
        if arm == "windowed":
            self.draft_windowed(log)
        elif arm == "native":
            self.draft_native(log)
        else:
            raise ValueError(arm)
        self.verify(log)
        self.accept(log)
        if log: log.mark(None)

    # ----------------------------------------------------------------------------- e2e
    _INPUTS = ("q_verify", "logits", "tokens", "q_ctx", "q_fwd", "k_ctx", "v_ctx", "k_fwd", "v_fwd")
    _OUTPUTS = ("accepted", "n_accepted")

    def pack_io(self):
        """Re-homes the per-step inputs and the acceptance outputs into one contiguous device
        buffer each (views at 256-byte offsets, contents kept), so that a step's host transfers
        are one copy in and one copy out."""
        b = self.b

        def pack(tensors):
            offs, total = [], 0
            for t in tensors:
                offs.append(total)
                total += (t.numel() * t.element_size() + 255) // 256 * 256
            buf = torch.empty(total, dtype=torch.uint8, device=tensors[0].device)
            views = []
            for t, o in zip(tensors, offs):
                v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                v.copy_(t)
                views.append(v)
            return buf, views

        self._in_buf, views = pack([getattr(b, n) for n in self._INPUTS])
        for n, v in zip(self._INPUTS, views):
            setattr(b, n, v)
        self._out_buf, views = pack([b.out[n] for n in self._OUTPUTS])
        for n, v in zip(self._OUTPUTS, views):
            b.out[n] = v

    def host_inputs(self) -> Dict[str, torch.Tensor]:
        """Pinned host copies of every per-step input (what a serving loop hands over): one
        buffer with the device layout after pack_io, else one tensor per input."""
        if getattr(self, "_in_buf", None) is not None:
            return {"packed_inputs": self._in_buf.cpu().pin_memory()}
        return {n: getattr(self.b, n).cpu().pin_memory() for n in self._INPUTS}

    def host_outputs(self) -> Dict[str, torch.Tensor]:
        if getattr(self, "_out_buf", None) is not None:
            return {"packed_outputs": torch.empty(self._out_buf.shape, dtype=torch.uint8).pin_memory()}
        b = self.b
        return {n: torch.empty(b.out[n].shape, dtype=b.out[n].dtype).pin_memory() for n in self._OUTPUTS}

    def run_e2e(self, arm: str, h_in: Dict[str, torch.Tensor], h_out: Dict[str, torch.Tensor]):
        """H2D of the step's inputs, the step, D2H of the accepted tokens (all async)."""
        b = self.b
        for n, t in h_in.items():
            (self._in_buf if n == "packed_inputs" else getattr(b, n)).copy_(t, non_blocking=True)
        self.run(arm)
        for n, t in h_out.items():
            t.copy_(self._out_buf if n == "packed_outputs" else b.out[n], non_blocking=True)

    @staticmethod
    def bytes_of(ts: Dict[str, torch.Tensor]) -> int:
        return sum(t.numel() * t.element_size() for t in ts.values())
