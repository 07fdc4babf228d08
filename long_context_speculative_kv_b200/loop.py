"""The speculative decode loop on the device: Windowed-MTP decode steps with real acceptance
decisions, rollback of rejected draft rows, and no host round trip between steps (so a step
can be captured once as a CUDA graph and replayed).

One step, in the order of the pages' cost identity (Pith verdict on arXiv 2607.21535,
pith_extraction.key_machinery, Eq. 1: t_step = t_verify + t_ctx_draft + gamma * t_fwd_draft):

  * draft context pass: the draft rows of the tokens the previous step committed go into the
    ring at the first rejected position (ring_kv_append_at: this is the rollback of the previous
    step's draft-forward rows), then one draft attention call with n_q = gamma + 1 (the worst
    case of the pages' accounting; queries before the newly committed ones re-read older
    positions);
  * gamma draft forwards: ring append of one row and draft attention with n_q = 1, one library
    call (draft_attn_window_append);
  * proposals: the synthetic draft head (tokens [B, gamma + 1], node 0 = last committed token);
  * verify: one verify_attn per target attention layer over T - 1 + gamma + 1 keys;
  * the synthetic target head's logits for the gamma + 1 nodes, accept_greedy, spec_commit.

The native arm runs draft_attn_full over the paged draft cache instead (kv_len T for the context
pass, T + j for forward j).  Each arm's draft K/V rows and every target layer's K/V are fixed
synthetic rows per position: the models that would produce them are not part of the path, and
the synthetic heads choose tokens without reading the attention outputs, so both arms commit
the same tokens (windowing changes only which tokens are proposed, never which are accepted
[AI field-notes abstract]; with these heads not even the proposals change).

The ring needs capacity >= n_sink + window + gamma: the draft forwards of a step overwrite the
gamma oldest slots, and after the rollback those slots hold window rows again.
"""
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import api
from .step import CallLog, StepBuffers


@dataclass
class LoopState:
    history: torch.Tensor       # [B, max_tokens] int32
    n_tokens: torch.Tensor      # [B] int64, committed tokens T
    append_pos: torch.Tensor    # [B] int64
    n_append: torch.Tensor      # [B] int32
    verify_len: torch.Tensor    # [B] int32  (T - 1 + n_q)
    draft_len: torch.Tensor     # [gamma + 1, B] int32  (T + j)

    @staticmethod
    def start(history: torch.Tensor, n_tokens: Sequence[int], gamma: int) -> "LoopState":
        """State before the first step.  ``history`` [B, max_tokens] int32 (device) holds the
        prompts, request b's in history[b, :n_tokens[b]].  The first context pass appends the
        draft row of each prompt's last token (the ring must already hold the ones before it)."""
        if history.dtype != torch.int32 or history.dim() != 2:
            raise TypeError("history must be a 2-d int32 tensor")
        B, max_tokens = history.shape
        if len(n_tokens) != B or not all(1 <= int(t) <= max_tokens for t in n_tokens):
            raise ValueError("prompt lengths must be in [1, max_tokens]")
        dev = history.device
        T = torch.tensor([int(t) for t in n_tokens], dtype=torch.int64, device=dev)
        n_q = gamma + 1
        return LoopState(
            history=history, n_tokens=T, append_pos=T - 1,
            n_append=torch.ones(B, dtype=torch.int32, device=dev),
            verify_len=(T - 1 + n_q).to(torch.int32),
            draft_len=torch.stack([(T + j).to(torch.int32) for j in range(gamma + 1)]).contiguous())


class DecodeLoop:
    def __init__(self, bufs: StepBuffers, gamma: int, state: LoopState, vocab: int,
                 target_seed: int, draft_seed: int, agree24: int):
        if bufs.tree_parent is not None:
            raise ValueError("the decode loop drafts chains")
        self.b, self.gamma, self.s = bufs, gamma, state
        self.vocab, self.target_seed, self.draft_seed, self.agree24 = vocab, target_seed, draft_seed, agree24
        self.n_layers = bufs.q_verify.shape[0]
        B, n_q = bufs.q_verify.shape[1:3]
        if n_q != gamma + 1:
            raise ValueError("verify queries must be gamma + 1")
        dev = bufs.q_verify.device
        self.tokens = torch.zeros((B, n_q), dtype=torch.int32, device=dev)
        self.logits = torch.empty((B, n_q, vocab), dtype=torch.float32, device=dev)
        self.accepted = torch.empty((B, n_q), dtype=torch.int32, device=dev)
        self.n_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
        o = bufs.out
        o["verify"] = torch.empty_like(bufs.q_verify[0])
        o["verify_lse"] = torch.empty(bufs.q_verify.shape[1:4], dtype=torch.float32, device=dev)
        o["ctx"] = torch.empty_like(bufs.q_ctx)
        o["ctx_lse"] = torch.empty(bufs.q_ctx.shape[:3], dtype=torch.float32, device=dev)
        o["fwd"] = torch.empty_like(bufs.q_fwd[0])
        o["fwd_lse"] = torch.empty(bufs.q_fwd.shape[1:4], dtype=torch.float32, device=dev)
        if bufs.ws is None:
            Hq = bufs.q_verify.shape[3]
            Hkv = bufs.k_pools[0].shape[1]
            bufs.ws = torch.zeros(max(api.workspace_bytes(B, n_q, Hq, Hkv), api.workspace_bytes(B, 1, Hq, Hkv)),
                                  dtype=torch.uint8, device=dev)
        if bufs.ring_k is not None and bufs.ring_k.shape[2] < bufs.n_sink + bufs.window + gamma:
            raise ValueError("ring capacity must be >= n_sink + window + gamma for the rollback")

    def draft_windowed(self, log: Optional[CallLog] = None):
        b, s = self.b, self.s
        if log: log.mark("append_ctx")
        api.ring_kv_append_at(b.ring_k, b.ring_v, b.ring_len, b.k_ctx, b.v_ctx, s.append_pos, s.n_append,
                              b.n_sink)
        if log: log.mark("window_ctx")
        api.draft_attn_window(b.q_ctx, b.ring_k, b.ring_v, b.ring_len, b.n_sink, b.window, b.sm_scale, b.ws,
                              out=b.out["ctx"], lse=b.out["ctx_lse"])
        for j in range(self.gamma):
            if log: log.mark("window_fwd")
            api.draft_attn_window_append(b.q_fwd[j], b.ring_k, b.ring_v, b.ring_len, b.k_fwd[j], b.v_fwd[j],
                                         b.n_sink, b.window, b.sm_scale, b.ws, out=b.out["fwd"],
                                         lse=b.out["fwd_lse"])

    def draft_native(self, log: Optional[CallLog] = None):
        b, s = self.b, self.s
        if log: log.mark("full_ctx")
        api.draft_attn_full(b.q_ctx, b.k_draft, b.v_draft, b.table_d, s.draft_len[0], b.sm_scale, b.ws,
                            out=b.out["ctx"], lse=b.out["ctx_lse"])
        for j in range(self.gamma):
            if log: log.mark("full_fwd")
            api.draft_attn_full(b.q_fwd[j], b.k_draft, b.v_draft, b.table_d, s.draft_len[j + 1], b.sm_scale,
                                b.ws, out=b.out["fwd"], lse=b.out["fwd_lse"])

    def step(self, arm: str, log: Optional[CallLog] = None):
        b, s = self.b, self.s
        if arm == "windowed":
            self.draft_windowed(log)
        elif arm == "native":
            self.draft_native(log)
        else:
            raise ValueError(arm)
        if log: log.mark("propose")
        api.synth_draft_tokens(s.history, s.n_tokens, self.gamma, self.vocab, self.target_seed,
                               self.draft_seed, self.agree24, tokens=self.tokens)
        for layer in range(self.n_layers):
            if log: log.mark("verify")
            api.verify_attn(b.q_verify[layer], b.k_pools[layer], b.v_pools[layer], b.table_v, s.verify_len,
                            b.sm_scale, b.ws, out=b.out["verify"], lse=b.out["verify_lse"])
        if log: log.mark("target_logits")
        api.synth_target_logits(s.history, s.n_tokens, self.tokens, self.vocab, self.target_seed,
                                logits=self.logits)
        if log: log.mark("accept")
        api.accept_greedy(self.logits, self.tokens, None, accepted=self.accepted, n_accepted=self.n_accepted)
        if log: log.mark("commit")
        api.spec_commit(self.accepted, self.n_accepted, s.history, s.n_tokens, s.append_pos, s.n_append,
                        verify_len=s.verify_len, n_q_verify=self.gamma + 1, draft_len=s.draft_len)
        if log: log.mark(None)
