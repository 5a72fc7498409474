"""Seeded synthetic inputs for the DSpark loss sweep.

This module only draws random numbers and lays tensors out; it holds none of the
loss arithmetic, so the CPU oracle and the CUDA path can both consume what it
makes without sharing any part of the method.

The shapes, value distributions and mask structure follow the Qwen3-8B DSpark
recipe (TorchSpec pull request #132: block_size 7, gamma 4.0, markov_rank 256,
vocab 151936) and the checkpoint contract of the NeMo RL design doc "DSpark
Auxiliary Heads" (markov_w1 [target_vocab, rank], markov_w2 [draft_vocab, rank],
confidence proj [1, hidden + rank]).  No dataset stands behind any of it.

Conventions taken for the inputs (they are readings, not measurements):
  * ``N(0, s)`` names a normal with standard deviation ``s``.
  * eval_mask is a contiguous prefix of per-block length L (drawn uniformly in
    the configuration's range); ``block_keep = (L >= 1)``.
  * target_ids are drawn from the categorical distribution of the target row
    (Gumbel-max on the rounded target logits).
  * prev_ids are anchor-seeded: slot 0 holds a uniform anchor token, slot k
    holds the label of slot k-1 (TorchSpec pull request #132, scope list).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

# Row count of one Qwen3 vocabulary (both Markov tables have this many rows in the
# pinned deepseek-ai/dspark_qwen3_8b_block7 artifact, NeMo RL "DSpark Auxiliary Heads").
QWEN3_VOCAB = 151936

CONFIGS = {
    # tiny fp32 case with given confidence logits
    "tiny": dict(B=1, N=2, K=4, V=1024, dtype="f32", prefix=(4, 4), conf="given",
                 markov=False, lm_head=False),
    # the Qwen3-8B recipe shape, no heads
    "recipe": dict(B=4, N=16, K=7, V=QWEN3_VOCAB, dtype="bf16", prefix=(1, 7), conf=None,
                   markov=False, lm_head=False),
    # recipe + Markov head (rank 256) + confidence head (hidden 4096, Markov-fused)
    "recipe_heads": dict(B=4, N=16, K=7, V=QWEN3_VOCAB, dtype="bf16", prefix=(1, 7),
                         conf="head", markov=True, lm_head=False),
    # recipe + heads, with the teacher computed from target final hidden states
    "lm_head_teacher": dict(B=4, N=16, K=7, V=QWEN3_VOCAB, dtype="bf16", prefix=(1, 7),
                            conf="head", markov=True, lm_head=True),
    # 8192 rows, ragged prefixes including empty blocks, heads on
    "large": dict(B=8, N=64, K=16, V=QWEN3_VOCAB, dtype="bf16", prefix=(0, 16),
                  conf="head", markov=True, lm_head=False),
}
CONFIG_ORDER = ["tiny", "recipe", "recipe_heads", "lm_head_teacher", "large"]

MARKOV_RANK = 256
HIDDEN = 4096


@dataclasses.dataclass
class DSparkInputs:
    """One synthetic micro-batch. Tensors are laid out [B, N, K(, V)] row-major."""

    B: int
    N: int
    K: int
    V: int
    dtype: str                                  # "f32" or "bf16" (draft/target/dlogits)
    draft_logits: torch.Tensor                  # [B,N,K,V]
    target_logits: Optional[torch.Tensor]       # [B,N,K,V] or None
    target_ids: torch.Tensor                    # int64 [B,N,K]
    eval_mask: torch.Tensor                     # uint8 [B,N,K]
    block_keep: Optional[torch.Tensor]          # uint8 [B,N]
    confidence_logits: Optional[torch.Tensor] = None   # float32 [B,N,K]
    prev_ids: Optional[torch.Tensor] = None     # int64 [B,N,K] (target vocabulary)
    valid: Optional[torch.Tensor] = None        # uint8 [B,N,K]
    markov_w1: Optional[torch.Tensor] = None    # bf16 [Vt, r]
    markov_w2: Optional[torch.Tensor] = None    # bf16 [V, r]
    draft_hidden: Optional[torch.Tensor] = None  # bf16 [B,N,K,H]
    conf_w: Optional[torch.Tensor] = None       # bf16 [1, H (+ r)]
    conf_b: Optional[torch.Tensor] = None       # float32 [1]
    conf_with_markov: bool = False
    target_hidden: Optional[torch.Tensor] = None  # bf16 [B,N,K,Ht]
    lm_head: Optional[torch.Tensor] = None      # bf16 [V, Ht]
    target_norm_weight: Optional[torch.Tensor] = None  # bf16 [Ht]: target_hidden is pre-norm
    target_norm_eps: float = 1e-6
    gamma: Optional[float] = 4.0
    ce_alpha: float = 0.1
    l1_alpha: float = 0.9
    conf_alpha: float = 1.0
    grad_scale: float = 1.0
    name: str = ""

    @property
    def R(self) -> int:
        return self.B * self.N * self.K

    def tensors(self):
        return {f.name: getattr(self, f.name) for f in dataclasses.fields(self)
                if isinstance(getattr(self, f.name), torch.Tensor)}

    def to(self, device) -> "DSparkInputs":
        kw = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return DSparkInputs(**kw)


def _normal(gen, shape, std, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).mul_(std).to(dtype)


def _gumbel_max_ids(gen, logits_rows: torch.Tensor, chunk: int = 256) -> torch.Tensor:
    """Draw one categorical sample per row of ``logits_rows`` (Gumbel-max)."""
    R, V = logits_rows.shape
    out = torch.empty(R, dtype=torch.int64, device=logits_rows.device)
    for r0 in range(0, R, chunk):
        x = logits_rows[r0:r0 + chunk].float()
        u = torch.rand(x.shape, generator=gen, device=x.device).clamp_(1e-12, 1.0 - 1e-7)
        out[r0:r0 + chunk] = torch.argmax(x - torch.log(-torch.log(u)), dim=-1)
    return out


def make_inputs(name: str = "recipe", device="cpu", seed: Optional[int] = None,
                **overrides) -> DSparkInputs:
    """Build the synthetic inputs of configuration ``name``.

    ``overrides`` may replace any of B, N, K, V, dtype, prefix (lo, hi), conf
    ("given" | "head" | None), markov, lm_head, plus: ``hidden`` (confidence-head
    hidden size), ``target_hidden_size``, ``rank``, ``target_vocab``,
    ``valid_p`` (probability a slot is Markov-valid), ``mask_holes`` (add stray
    ones after each prefix so the cumprod inside the loss has work to do),
    ``no_target`` (CE-only), ``gamma``, ``grad_scale``, ``conf_with_markov``,
    ``markov_std`` (std of both Markov tables; 0.02 is the initialisation scale, a
    larger one makes the correction visible in tests), ``conf_bias``,
    ``target_prenorm`` (teacher hidden states drawn before the target's final RMS norm:
    N(0, 4) with a norm weight N(1, 0.1) and eps 1e-6; the labels are drawn from the
    normed teacher).
    The default seed is 1234 + the configuration's index.
    """
    base = dict(CONFIGS[name])
    base.update(dict(hidden=HIDDEN, target_hidden_size=HIDDEN, rank=MARKOV_RANK,
                     target_vocab=None, valid_p=0.9, mask_holes=False, no_target=False,
                     gamma=4.0, grad_scale=1.0, conf_with_markov=None, markov_std=0.02,
                     conf_bias=0.0, target_prenorm=False))
    unknown = set(overrides) - set(base)
    if unknown:
        raise TypeError(f"unknown overrides {sorted(unknown)}")
    base.update(overrides)
    c = base
    if seed is None:
        seed = 1234 + CONFIG_ORDER.index(name)
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    B, N, K, V = c["B"], c["N"], c["K"], c["V"]
    R = B * N * K
    ldt = torch.float32 if c["dtype"] == "f32" else torch.bfloat16
    Vt = c["target_vocab"] or V

    # ---- prefix masks -------------------------------------------------------
    lo, hi = c["prefix"]
    L = torch.randint(lo, hi + 1, (B, N), generator=gen, device=device)
    kk = torch.arange(K, device=device)
    eval_mask = (kk.view(1, 1, K) < L.view(B, N, 1)).to(torch.uint8)
    if c["mask_holes"]:
        stray = torch.rand((B, N, K), generator=gen, device=device) < 0.5
        eval_mask = torch.where(stray, torch.ones_like(eval_mask), eval_mask)
    block_keep = (L >= 1).to(torch.uint8)

    # ---- logits --------------------------------------------------------------
    lm_head = target_hidden = None
    if c["dtype"] == "f32":
        draft = _normal(gen, (B, N, K, V), 2.0, device)
        target = draft + _normal(gen, (B, N, K, V), 1.0, device)
    else:
        draft = _normal(gen, (B, N, K, V), 3.0, device, torch.bfloat16)
        target = (0.8 * draft.float() + _normal(gen, (B, N, K, V), 1.5, device)).to(torch.bfloat16)
    norm_w = None
    if c["lm_head"]:
        Ht = c["target_hidden_size"]
        target_hidden = _normal(gen, (B, N, K, Ht), 4.0 if c["target_prenorm"] else 1.0, device, torch.bfloat16)
        lm_head = _normal(gen, (V, Ht), 0.02, device, torch.bfloat16)
        # the teacher rows only serve to draw labels here; the loss recomputes them
        teacher = torch.empty((R, V), dtype=torch.float32, device=device)
        h2 = target_hidden.reshape(R, Ht).float()
        if c["target_prenorm"]:
            norm_w = (1.0 + _normal(gen, (Ht,), 0.1, device)).to(torch.bfloat16)
            h2 = h2 * torch.rsqrt(h2.pow(2).mean(-1, keepdim=True) + 1e-6) * norm_w.float()
        w = lm_head.float()
        for r0 in range(0, R, 64):
            teacher[r0:r0 + 64] = h2[r0:r0 + 64] @ w.t()
        ids = _gumbel_max_ids(gen, teacher)
        del teacher
        target = None
    elif c["no_target"]:
        ids = _gumbel_max_ids(gen, draft.reshape(R, V))
        target = None
    else:
        ids = _gumbel_max_ids(gen, target.reshape(R, V))
    target_ids = ids.view(B, N, K)

    inp = DSparkInputs(B=B, N=N, K=K, V=V, dtype=c["dtype"], draft_logits=draft,
                       target_logits=target, target_ids=target_ids, eval_mask=eval_mask,
                       block_keep=block_keep, gamma=c["gamma"], grad_scale=c["grad_scale"],
                       name=name, target_hidden=target_hidden, lm_head=lm_head,
                       target_norm_weight=norm_w)

    # ---- Markov head ---------------------------------------------------------
    r = c["rank"]
    if c["markov"]:
        anchor = torch.randint(0, Vt, (B, N, 1), generator=gen, device=device)
        ids_in_t = target_ids.clamp(max=Vt - 1)
        inp.prev_ids = torch.cat([anchor, ids_in_t[..., :-1]], dim=-1).contiguous()
        inp.valid = (torch.rand((B, N, K), generator=gen, device=device) < c["valid_p"]).to(torch.uint8)
        inp.markov_w1 = _normal(gen, (Vt, r), c["markov_std"], device, torch.bfloat16)
        inp.markov_w2 = _normal(gen, (V, r), c["markov_std"], device, torch.bfloat16)

    # ---- confidence ----------------------------------------------------------
    if c["conf"] == "given":
        inp.confidence_logits = _normal(gen, (B, N, K), 1.0, device)
    elif c["conf"] == "head":
        H = c["hidden"]
        with_markov = c["conf_with_markov"]
        if with_markov is None:
            with_markov = bool(c["markov"])
        inp.conf_with_markov = with_markov
        inp.draft_hidden = _normal(gen, (B, N, K, H), 1.0, device, torch.bfloat16)
        inp.conf_w = _normal(gen, (1, H + (r if with_markov else 0)), 0.02, device, torch.bfloat16)
        inp.conf_b = torch.full((1,), float(c["conf_bias"]), dtype=torch.float32, device=device)
        if not c["markov"]:
            # a confidence head without a Markov head still needs the valid-slot mask
            inp.valid = (torch.rand((B, N, K), generator=gen, device=device) < c["valid_p"]).to(torch.uint8)
    return inp
