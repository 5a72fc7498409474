"""PyTorch-facing wrapper of the C ABI: builds the ABI structs from CUDA tensors,
allocates the outputs with torch, and calls the library on the current stream.

Argument marshalling only.  Nothing here computes any part of the loss.
"""

from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import abi
from .synthetic import DSparkInputs


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: Optional[torch.Tensor], dtype, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def problem_struct(inp: DSparkInputs) -> abi.dspark_problem_t:
    """The dspark_problem_t describing ``inp`` (tensors must stay alive)."""
    ldt = torch.float32 if inp.dtype == "f32" else torch.bfloat16
    p = abi.dspark_problem_t()
    p.B, p.N, p.K, p.V = inp.B, inp.N, inp.K, inp.V
    p.logits_dtype = abi.DSPARK_F32 if inp.dtype == "f32" else abi.DSPARK_BF16
    d = _need(inp.draft_logits, ldt, "draft_logits")
    p.draft_logits, p.draft_ld = _ptr(d), inp.V
    if inp.target_logits is not None:
        p.target_logits = _ptr(_need(inp.target_logits, ldt, "target_logits"))
        p.target_ld = inp.V
    p.target_ids = _ptr(_need(inp.target_ids, torch.int64, "target_ids"))
    p.eval_mask = _ptr(_need(inp.eval_mask, torch.uint8, "eval_mask"))
    p.block_keep = _ptr(_need(inp.block_keep, torch.uint8, "block_keep"))
    p.confidence_logits = _ptr(_need(inp.confidence_logits, torch.float32, "confidence_logits"))
    if inp.lm_head is not None:
        p.target_hidden = _ptr(_need(inp.target_hidden, torch.bfloat16, "target_hidden"))
        p.lm_head = _ptr(_need(inp.lm_head, torch.bfloat16, "lm_head"))
        p.target_hidden_size = inp.lm_head.shape[1]
        if inp.target_norm_weight is not None:
            p.target_norm_weight = _ptr(_need(inp.target_norm_weight, torch.bfloat16, "target_norm_weight"))
            p.target_norm_eps = float(inp.target_norm_eps)
    if inp.markov_w2 is not None:
        p.prev_ids = _ptr(_need(inp.prev_ids, torch.int64, "prev_ids"))
        p.markov_w1 = _ptr(_need(inp.markov_w1, torch.bfloat16, "markov_w1"))
        p.markov_w2 = _ptr(_need(inp.markov_w2, torch.bfloat16, "markov_w2"))
        p.target_vocab = inp.markov_w1.shape[0]
        p.markov_rank = inp.markov_w2.shape[1]
    if inp.valid is not None:
        p.valid = _ptr(_need(inp.valid, torch.uint8, "valid"))
    if inp.conf_w is not None:
        p.draft_hidden = _ptr(_need(inp.draft_hidden, torch.bfloat16, "draft_hidden"))
        p.hidden_size = inp.draft_hidden.shape[-1]
        p.conf_w = _ptr(_need(inp.conf_w, torch.bfloat16, "conf_w"))
        p.conf_b = _ptr(_need(inp.conf_b, torch.float32, "conf_b"))
        p.conf_with_markov = 1 if inp.conf_with_markov else 0
    return p


def params_struct(inp: DSparkInputs, invalid_row_mode: int = 0) -> abi.dspark_params_t:
    prm = abi.dspark_params_t()
    prm.ce_alpha, prm.l1_alpha, prm.conf_alpha = inp.ce_alpha, inp.l1_alpha, inp.conf_alpha
    if inp.target_logits is None and inp.lm_head is None:
        prm.l1_alpha = 0.0
    prm.gamma = inp.gamma if inp.gamma is not None else 1.0
    prm.gamma_enabled = 0 if inp.gamma is None else 1
    prm.invalid_row_mode = invalid_row_mode
    return prm


def workspace_bytes(inp: DSparkInputs) -> int:
    p = problem_struct(inp)
    return int(abi.dspark_workspace_size(ctypes.byref(p)))


def new_workspace(inp: DSparkInputs) -> torch.Tensor:
    n = workspace_bytes(inp)
    return torch.empty(n + 256, dtype=torch.uint8, device=inp.draft_logits.device)


def _aligned_ws(ws: torch.Tensor):
    base = ws.data_ptr()
    off = (-base) % 256
    return ctypes.c_void_p(base + off), ws.numel() - off


class Outputs:
    """Device buffers one fused call writes (allocated once, reusable)."""

    def __init__(self, inp: DSparkInputs, rows: bool = True, grads: bool = True):
        dev = inp.draft_logits.device
        R = inp.R
        f32 = dict(dtype=torch.float32, device=dev)
        self.loss_num = torch.zeros(1, **f32)
        self.num_tokens = torch.zeros(1, dtype=torch.int64, device=dev)
        self.report = torch.zeros(abi.DSPARK_REP_COUNT, 2, **f32)
        self.ce_rows = torch.zeros(R, **f32) if rows else None
        self.l1_rows = torch.zeros(R, **f32) if rows else None
        self.accept_rows = torch.zeros(R, **f32) if rows else None
        self.conf_rows = torch.zeros(R, **f32) if rows else None
        self.grad_scale = torch.full((1,), float(inp.grad_scale), **f32)
        self.dlogits = torch.empty_like(inp.draft_logits) if grads else None
        self.dconf = torch.zeros(R, **f32) if grads else None
        self.dW1 = self.dW2 = self.dconf_w = self.dconf_b = self.dhidden = None
        if grads and inp.markov_w2 is not None:
            self.dW1 = torch.zeros(inp.markov_w1.shape, **f32)
            self.dW2 = torch.zeros(inp.markov_w2.shape, **f32)
        if grads and inp.conf_w is not None:
            self.dconf_w = torch.zeros(inp.conf_w.numel(), **f32)
            self.dconf_b = torch.zeros(1, **f32)
            self.dhidden = torch.zeros(inp.draft_hidden.shape, dtype=torch.bfloat16, device=dev)
        self.ws = new_workspace(inp)

    def fwd_struct(self) -> abi.dspark_fwd_out_t:
        o = abi.dspark_fwd_out_t()
        o.loss_num, o.num_tokens, o.report = _ptr(self.loss_num), _ptr(self.num_tokens), _ptr(self.report)
        o.ce_rows, o.l1_rows = _ptr(self.ce_rows), _ptr(self.l1_rows)
        o.accept_rows, o.conf_rows = _ptr(self.accept_rows), _ptr(self.conf_rows)
        return o

    def grads_struct(self, inp: DSparkInputs, accumulate: bool = False) -> abi.dspark_grads_t:
        g = abi.dspark_grads_t()
        g.grad_scale = _ptr(self.grad_scale)
        g.dlogits, g.dlogits_ld = _ptr(self.dlogits), inp.V
        g.dconf = _ptr(self.dconf)
        g.dW1, g.dW2 = _ptr(self.dW1), _ptr(self.dW2)
        g.dconf_w, g.dconf_b, g.dhidden = _ptr(self.dconf_w), _ptr(self.dconf_b), _ptr(self.dhidden)
        g.accumulate = 1 if accumulate else 0
        return g


class Call:
    """A prepared fused forward+backward call: structs built once, launched many times."""

    def __init__(self, inp: DSparkInputs, out: Optional[Outputs] = None, grads: bool = True,
                 rows: bool = True, invalid_row_mode: int = 0, accumulate: bool = False):
        self.inp = inp
        self.out = out if out is not None else Outputs(inp, rows=rows, grads=grads)
        self.prob = problem_struct(inp)
        self.prm = params_struct(inp, invalid_row_mode)
        self.fwd = self.out.fwd_struct()
        self.grads = self.out.grads_struct(inp, accumulate) if grads else None
        self.ws_ptr, self.ws_len = _aligned_ws(self.out.ws)

    def launch(self, stream=None) -> None:
        s = torch.cuda.current_stream().cuda_stream if stream is None else stream
        st = abi.dspark_loss_fwd(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.fwd),
                                 ctypes.byref(self.grads) if self.grads is not None else None,
                                 self.ws_ptr, self.ws_len, ctypes.c_void_p(s))
        abi.check(st, "dspark_loss_fwd")

    def backward(self, stream=None) -> None:
        s = torch.cuda.current_stream().cuda_stream if stream is None else stream
        st = abi.dspark_loss_bwd(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.grads),
                                 self.ws_ptr, self.ws_len, ctypes.c_void_p(s))
        abi.check(st, "dspark_loss_bwd")

    def check_status(self, stream=None) -> int:
        s = torch.cuda.current_stream().cuda_stream if stream is None else stream
        return int(abi.dspark_check_status(self.ws_ptr, ctypes.c_void_p(s)))


def dspark_loss(inp: DSparkInputs, grads: bool = True, rows: bool = True, invalid_row_mode: int = 0):
    """One fused call on the current stream; returns the Outputs (not synchronised)."""
    c = Call(inp, grads=grads, rows=rows, invalid_row_mode=invalid_row_mode)
    c.launch()
    return c.out


def acceptance(l1_rows: torch.Tensor, eval_mask: torch.Tensor, block_keep: Optional[torch.Tensor] = None):
    """Standalone acceptance report: (accept_pair[2], tau_pair[2], accept_rows[R])."""
    B, N, K = eval_mask.shape
    dev = l1_rows.device
    _need(l1_rows, torch.float32, "l1_rows")
    _need(eval_mask, torch.uint8, "eval_mask")
    _need(block_keep, torch.uint8, "block_keep")
    ap = torch.zeros(2, dtype=torch.float32, device=dev)
    tp = torch.zeros(2, dtype=torch.float32, device=dev)
    ar = torch.zeros(B * N * K, dtype=torch.float32, device=dev)
    st = abi.dspark_acceptance(B, N, K, _ptr(l1_rows), _ptr(eval_mask), _ptr(block_keep), _ptr(ap),
                               _ptr(tp), _ptr(ar), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    abi.check(st, "dspark_acceptance")
    return ap, tp, ar


# ------------------------------------------------------- data-parallel reduction
REPORT_VECTOR_LEN = 2 + 2 * abi.DSPARK_REP_COUNT


def reduce_report(loss_num: torch.Tensor, num_tokens: torch.Tensor, report: torch.Tensor, group=None):
    """Sum one micro-batch's forward outputs over the data-parallel ranks of ``group``:
    the numerator, the supervised-token count and the report pairs, packed into one FP64
    vector [loss_num, num_tokens, num_0, den_0, ..., num_5, den_5] and all-reduced (SUM)
    in a single collective.  Nothing is divided: the caller forms each ratio once, from
    the sums (the Megatron-Bridge API doc's Return contract).  Counts and denominators
    are integers below 2^53, so their FP64 sums are exact.  Works on CUDA tensors over
    NCCL and on CPU tensors over gloo; returns (loss_num [1] f64, num_tokens [1] i64,
    report [DSPARK_REP_COUNT, 2] f64) on the inputs' device."""
    import torch.distributed as dist
    if report.numel() != 2 * abi.DSPARK_REP_COUNT:
        raise ValueError(f"report must hold {2 * abi.DSPARK_REP_COUNT} values")
    vec = torch.cat([loss_num.reshape(1).to(torch.float64), num_tokens.reshape(1).to(torch.float64),
                     report.reshape(-1).to(torch.float64)])
    dist.all_reduce(vec, op=dist.ReduceOp.SUM, group=group)
    return vec[:1], vec[1:2].to(torch.int64), vec[2:].reshape(abi.DSPARK_REP_COUNT, 2)


# ------------------------------------------------------- vocabulary-parallel path
def even_shards(V: int, tp_size: int, align: int) -> list:
    """Bounds [0, v_1, ..., V] of tp_size contiguous vocabulary shards whose widths are
    multiples of ``align`` columns (8 bf16 / 4 fp32: the 16-byte rule), as even as
    that allows (the first shards take the remainder)."""
    if V % align or tp_size < 1 or V // align < tp_size:
        raise ValueError("V must be a multiple of align, with at least one vector of align columns per rank")
    base, extra = divmod(V // align, tp_size)
    bounds = [0]
    for k in range(tp_size):
        bounds.append(bounds[-1] + (base + (1 if k < extra else 0)) * align)
    return bounds


class TPRank:
    """One tensor-parallel rank's calls (dspark_tp_partials, dspark_tp_l1,
    dspark_tp_finish, and with a head dspark_tp_heads_bwd) on its vocabulary shard of a
    micro-batch.

    ``inp`` holds rows that contain this rank's shard at columns [col0, col0 + width):
    the full rows (single-device emulation of a group) or just the shard (one rank per
    GPU, col0 = 0).  The shard is addressed in place, with the rows' stride; so are the
    shard's rows of ``inp.markov_w2`` and ``inp.lm_head`` (rows col0 .. col0 + width).
    dlogits of the shard go to the same columns of ``dlogits`` (rows shaped like
    ``inp``'s), and dW2 of the
    shard to the same rows of ``dW2`` (shaped like ``inp.markov_w2``), or to buffers this
    rank allocates.  Every rank writes its own copy of the forward outputs and of the
    replicated gradients (dW1, dconf_w, dconf_b, dhidden).
    """

    def __init__(self, inp: DSparkInputs, tp_size: int, vocab_begin: int, vocab_size: int,
                 col0: int = 0, width: Optional[int] = None, dlogits: Optional[torch.Tensor] = None,
                 dW2: Optional[torch.Tensor] = None, grads: bool = True, rows: bool = True,
                 invalid_row_mode: int = 0):
        dev = inp.draft_logits.device
        R = inp.R
        es = 4 if inp.dtype == "f32" else 2
        width = inp.V - col0 if width is None else width
        self.inp, self.col0, self.width = inp, col0, width
        p = problem_struct(inp)
        p.V = width
        p.draft_logits = ctypes.c_void_p(inp.draft_logits.data_ptr() + col0 * es)
        if inp.target_logits is not None:
            p.target_logits = ctypes.c_void_p(inp.target_logits.data_ptr() + col0 * es)
        markov = inp.markov_w2 is not None
        rank_ = inp.markov_w2.shape[1] if markov else 0
        if markov:
            p.markov_w2 = ctypes.c_void_p(inp.markov_w2.data_ptr() + col0 * rank_ * 2)
        if inp.lm_head is not None:  # the teacher from hidden states: this shard's lm_head rows
            p.lm_head = ctypes.c_void_p(inp.lm_head.data_ptr() + col0 * inp.lm_head.shape[1] * 2)
        self.prob = p
        self.prm = params_struct(inp, invalid_row_mode)
        self.tp = abi.dspark_tp_t(tp_size, vocab_begin, vocab_size)
        f32 = dict(dtype=torch.float32, device=dev)
        self.rec1 = torch.empty(R, abi.DSPARK_TP_REC1_FLOATS, **f32)
        self.rec2 = torch.empty(R, abi.DSPARK_TP_REC2_FLOATS, **f32)
        self.loss_num = torch.zeros(1, **f32)
        self.num_tokens = torch.zeros(1, dtype=torch.int64, device=dev)
        self.report = torch.zeros(abi.DSPARK_REP_COUNT, 2, **f32)
        self.ce_rows = torch.zeros(R, **f32) if rows else None
        self.l1_rows = torch.zeros(R, **f32) if rows else None
        self.accept_rows = torch.zeros(R, **f32) if rows else None
        self.conf_rows = torch.zeros(R, **f32) if rows else None
        self.grad_scale = torch.full((1,), float(inp.grad_scale), **f32)
        self.dconf = torch.zeros(R, **f32) if grads else None
        if grads and dlogits is None:
            dlogits = torch.zeros_like(inp.draft_logits)
        self.dlogits = dlogits if grads else None
        self.dW1 = self.dW2 = self.dconf_w = self.dconf_b = self.dhidden = self.de_part = None
        if grads and markov:
            self.dW1 = torch.zeros(inp.markov_w1.shape, **f32)
            self.dW2 = torch.zeros(inp.markov_w2.shape, **f32) if dW2 is None else dW2
            self.de_part = torch.zeros(R, rank_, **f32)
        if grads and inp.conf_w is not None:
            self.dconf_w = torch.zeros(inp.conf_w.numel(), **f32)
            self.dconf_b = torch.zeros(1, **f32)
            self.dhidden = torch.zeros(inp.draft_hidden.shape, dtype=torch.bfloat16, device=dev)
        o = abi.dspark_fwd_out_t()
        o.loss_num, o.num_tokens, o.report = _ptr(self.loss_num), _ptr(self.num_tokens), _ptr(self.report)
        o.ce_rows, o.l1_rows = _ptr(self.ce_rows), _ptr(self.l1_rows)
        o.accept_rows, o.conf_rows = _ptr(self.accept_rows), _ptr(self.conf_rows)
        self.fwd = o
        self.grads = None
        if grads:
            g = abi.dspark_grads_t()
            g.grad_scale = _ptr(self.grad_scale)
            g.dlogits = ctypes.c_void_p(self.dlogits.data_ptr() + col0 * es)
            g.dlogits_ld = inp.V
            g.dconf = _ptr(self.dconf)
            g.dW1 = _ptr(self.dW1)
            if self.dW2 is not None:
                g.dW2 = ctypes.c_void_p(self.dW2.data_ptr() + col0 * rank_ * 4)
            g.dconf_w, g.dconf_b, g.dhidden = _ptr(self.dconf_w), _ptr(self.dconf_b), _ptr(self.dhidden)
            self.grads = g
        self.has_heads = markov or inp.conf_w is not None
        self.ws = new_workspace(inp)
        self.ws_ptr, self.ws_len = _aligned_ws(self.ws)

    @staticmethod
    def _stream(stream):
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream if stream is None else stream)

    def partials(self, stream=None) -> torch.Tensor:
        st = abi.dspark_tp_partials(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.tp),
                                    _ptr(self.rec1), self.ws_ptr, self.ws_len, self._stream(stream))
        abi.check(st, "dspark_tp_partials")
        return self.rec1

    def l1(self, rec1_all: torch.Tensor, stream=None) -> torch.Tensor:
        _need(rec1_all, torch.float32, "rec1_all")
        st = abi.dspark_tp_l1(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.tp),
                              _ptr(rec1_all), _ptr(self.rec2), self.ws_ptr, self.ws_len, self._stream(stream))
        abi.check(st, "dspark_tp_l1")
        return self.rec2

    def finish(self, rec2_all: torch.Tensor, stream=None) -> None:
        _need(rec2_all, torch.float32, "rec2_all")
        st = abi.dspark_tp_finish(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.tp),
                                  _ptr(rec2_all), ctypes.byref(self.fwd),
                                  ctypes.byref(self.grads) if self.grads is not None else None,
                                  _ptr(self.de_part), self.ws_ptr, self.ws_len, self._stream(stream))
        abi.check(st, "dspark_tp_finish")
        return self.de_part

    def heads_bwd(self, de_all: Optional[torch.Tensor], stream=None) -> None:
        if self.grads is None:
            raise ValueError("this rank was built without gradients")
        _need(de_all, torch.float32, "de_all")
        st = abi.dspark_tp_heads_bwd(ctypes.byref(self.prob), ctypes.byref(self.prm), ctypes.byref(self.tp),
                                     _ptr(de_all), ctypes.byref(self.grads), self.ws_ptr, self.ws_len,
                                     self._stream(stream))
        abi.check(st, "dspark_tp_heads_bwd")

    def run(self, exchange) -> None:
        """The calls, with ``exchange`` (this rank's records -> every rank's records
        stacked in rank order, e.g. ``tp_exchange``) after each of the first two and, with
        the Markov head, after the third."""
        rec1_all = exchange(self.partials())
        de_part = self.finish(exchange(self.l1(rec1_all)))
        if self.grads is not None and self.has_heads:
            self.heads_bwd(exchange(de_part) if de_part is not None else None)

    def check_status(self, stream=None) -> int:
        return int(abi.dspark_check_status(self.ws_ptr, self._stream(stream)))


def tp_exchange(local: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's records in rank order, [world, *local.shape]: an all-gather over the
    tensor-parallel process group (NCCL for CUDA tensors)."""
    import torch.distributed as dist
    parts = [torch.empty_like(local) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.stack(parts)


def tp_group_emulated(inp: DSparkInputs, tp_size: int, grads: bool = True, rows: bool = True,
                      invalid_row_mode: int = 0) -> list:
    """A whole tensor-parallel group on this device: tp_size ranks over even shards of
    ``inp``'s full rows, stepped together, the exchange being a stack of the ranks'
    records (what the all-gather delivers).  The ranks share one dlogits buffer, each
    writing its own columns.  Returns the ranks (launched, not synchronised)."""
    align = 4 if inp.dtype == "f32" else 8
    bounds = even_shards(inp.V, tp_size, align)
    dl = torch.zeros_like(inp.draft_logits) if grads else None
    dw2 = torch.zeros(inp.markov_w2.shape, dtype=torch.float32, device=inp.draft_logits.device) \
        if (grads and inp.markov_w2 is not None) else None
    ranks = [TPRank(inp, tp_size, bounds[k], inp.V, col0=bounds[k], width=bounds[k + 1] - bounds[k],
                    dlogits=dl, dW2=dw2, grads=grads, rows=rows, invalid_row_mode=invalid_row_mode)
             for k in range(tp_size)]
    rec1_all = torch.stack([r.partials() for r in ranks])
    rec2_all = torch.stack([r.l1(rec1_all) for r in ranks])
    parts = [r.finish(rec2_all) for r in ranks]
    if grads and ranks[0].has_heads:
        de_all = torch.stack(parts) if parts[0] is not None else None
        for r in ranks:
            r.heads_bwd(de_all)
    return ranks
