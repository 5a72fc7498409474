"""Host-side checks of the C-ABI library: it loads, exports every symbol include/dspark.h
declares, its structs have the layout the ctypes binding assumes, and host validation
returns the documented status codes before touching the GPU.  No CUDA call is made."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dspark.h")


@pytest.fixture(scope="module")
def abi():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    from speculative_decoding_draft_vocab_b200 import abi as _abi
    return _abi


def _declared_functions():
    text = open(HEADER).read()
    return re.findall(r"DSPARK_API\s+[\w\s\*]+?\b(dspark_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(abi):
    names = _declared_functions()
    assert len(names) >= 6
    for n in names:
        assert hasattr(abi.lib, n), n
        assert hasattr(abi, n), f"binding lacks {n}"


C_LAYOUT = r"""
#include <stdio.h>
#include <stddef.h>
#include "dspark.h"
#define F(T, f) printf(#T " " #f " %zu\n", offsetof(T, f));
#define S(T) printf(#T " sizeof %zu\n", sizeof(T));
int main(void) {
BODY
  return 0;
}
"""


def test_struct_layout_matches_ctypes(abi):
    lines = []
    for cls in (abi.dspark_problem_t, abi.dspark_params_t, abi.dspark_fwd_out_t, abi.dspark_grads_t,
                abi.dspark_tp_t):
        t = cls.__name__
        lines.append(f"  S({t})")
        for f, _ in cls._fields_:
            lines.append(f"  F({t}, {f})")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        with open(src, "w") as f:
            f.write(C_LAYOUT.replace("BODY", "\n".join(lines)))
        subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    got = {}
    for line in out.splitlines():
        t, f, v = line.split()
        got[(t, f)] = int(v)
    for cls in (abi.dspark_problem_t, abi.dspark_params_t, abi.dspark_fwd_out_t, abi.dspark_grads_t,
                abi.dspark_tp_t):
        t = cls.__name__
        assert got[(t, "sizeof")] == ctypes.sizeof(cls), t
        for f, _ in cls._fields_:
            assert got[(t, f)] == getattr(cls, f).offset, (t, f)


def _problem(abi, V=1024, dtype=None, target=True):
    p = abi.dspark_problem_t()
    p.B, p.N, p.K, p.V = 1, 2, 4, V
    p.logits_dtype = abi.DSPARK_BF16 if dtype is None else dtype
    p.draft_logits, p.draft_ld = ctypes.c_void_p(0x10000), V
    if target:
        p.target_logits, p.target_ld = ctypes.c_void_p(0x20000), V
    p.target_ids = ctypes.c_void_p(0x30000)
    p.eval_mask = ctypes.c_void_p(0x40000)
    return p


def _params(abi, l1=0.9):
    prm = abi.dspark_params_t()
    prm.ce_alpha, prm.l1_alpha, prm.conf_alpha, prm.gamma = 0.1, l1, 1.0, 4.0
    prm.gamma_enabled = 1
    return prm


def _fwd(abi, p, prm, ws=0x100000, ws_bytes=1 << 30, grads=None):
    out = abi.dspark_fwd_out_t()
    return abi.dspark_loss_fwd(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(out),
                               ctypes.byref(grads) if grads is not None else None,
                               ctypes.c_void_p(ws), ws_bytes, None)


def test_host_validation_status_codes(abi):
    prm = _params(abi)
    # a teacher-dependent term without the teacher is refused before launch
    assert _fwd(abi, _problem(abi, target=False), prm) == abi.DSPARK_ERR_MISSING_TARGET
    # V * sizeof(bf16) not a multiple of 16 bytes
    assert _fwd(abi, _problem(abi, V=1020), prm) == abi.DSPARK_ERR_ALIGNMENT
    # misaligned row pointer
    p = _problem(abi)
    p.draft_logits = ctypes.c_void_p(0x10008)
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_ALIGNMENT
    # short workspace, missing workspace, misaligned workspace
    p = _problem(abi)
    assert _fwd(abi, p, prm, ws_bytes=16) == abi.DSPARK_ERR_WORKSPACE
    assert _fwd(abi, p, prm, ws=0) == abi.DSPARK_ERR_WORKSPACE
    assert _fwd(abi, p, prm, ws=0x100010) == abi.DSPARK_ERR_ALIGNMENT
    # bad sizes / dtype
    p = _problem(abi)
    p.K = 0
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    p = _problem(abi, dtype=7)
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # both confidence sources at once
    p = _problem(abi)
    p.confidence_logits = ctypes.c_void_p(0x50000)
    p.conf_w = ctypes.c_void_p(0x60000)
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # gamma enabled but not positive
    prm2 = _params(abi)
    prm2.gamma = 0.0
    assert _fwd(abi, _problem(abi), prm2) == abi.DSPARK_ERR_INVALID_ARG
    # a misaligned dlogits stride
    g = abi.dspark_grads_t()
    g.dlogits, g.dlogits_ld = ctypes.c_void_p(0x70000), 1028
    assert _fwd(abi, _problem(abi), prm, grads=g) == abi.DSPARK_ERR_ALIGNMENT
    # acceptance with NULL inputs
    assert abi.dspark_acceptance(1, 1, 1, None, None, None, None, None, None, None) == abi.DSPARK_ERR_INVALID_ARG
    assert abi.dspark_check_status(None, None) == abi.DSPARK_ERR_WORKSPACE


def test_status_strings_and_workspace_size(abi):
    for s in range(9):
        assert abi.dspark_status_string(s)
    p = _problem(abi)
    n1 = abi.dspark_workspace_size(ctypes.byref(p))
    p.N = 200
    n2 = abi.dspark_workspace_size(ctypes.byref(p))
    assert 0 < n1 < n2 and n1 % 256 == 0
    p.K = 0
    assert abi.dspark_workspace_size(ctypes.byref(p)) == 0


def _with_markov(abi, p, rank=64):
    p.prev_ids = ctypes.c_void_p(0x80000)
    p.valid = ctypes.c_void_p(0x90000)
    p.target_vocab = 500
    p.markov_w1 = ctypes.c_void_p(0xa0000)
    p.markov_w2 = ctypes.c_void_p(0xb0000)
    p.markov_rank = rank
    return p


def _with_conf_head(abi, p, H=256, with_markov=0):
    p.valid = ctypes.c_void_p(0x90000)
    p.draft_hidden = ctypes.c_void_p(0xc0000)
    p.hidden_size = H
    p.conf_w = ctypes.c_void_p(0xd0000)
    p.conf_b = ctypes.c_void_p(0xe0000)
    p.conf_with_markov = with_markov
    return p


def test_head_validation_status_codes(abi):
    prm = _params(abi)
    # the Markov head needs bf16 logits (its backward contracts bf16 dlogits)
    assert _fwd(abi, _with_markov(abi, _problem(abi, dtype=abi.DSPARK_F32)), prm) == abi.DSPARK_ERR_UNSUPPORTED
    # rank not a multiple of 8, misaligned table
    assert _fwd(abi, _with_markov(abi, _problem(abi), rank=60), prm) == abi.DSPARK_ERR_ALIGNMENT
    p = _with_markov(abi, _problem(abi))
    p.markov_w2 = ctypes.c_void_p(0xb0008)
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_ALIGNMENT
    # a partial Markov head (no valid mask / no W1) is refused
    p = _with_markov(abi, _problem(abi))
    p.valid = None
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    p = _with_markov(abi, _problem(abi))
    p.markov_w1 = None
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # confidence head: hidden size rule, a Markov input without the Markov head
    assert _fwd(abi, _with_conf_head(abi, _problem(abi), H=100), prm) == abi.DSPARK_ERR_ALIGNMENT
    assert _fwd(abi, _with_conf_head(abi, _problem(abi), with_markov=1), prm) == abi.DSPARK_ERR_INVALID_ARG
    p = _with_conf_head(abi, _problem(abi))
    p.conf_b = None
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # the confidence head needs the teacher (its label is 1 - L1/2)
    assert _fwd(abi, _with_conf_head(abi, _problem(abi, target=False)), _params(abi, l1=0.0)) == \
        abi.DSPARK_ERR_MISSING_TARGET


def test_markov_workspace_holds_corrected_rows(abi):
    p = _problem(abi, V=4096)
    p.B, p.N, p.K = 2, 3, 7
    base = abi.dspark_workspace_size(ctypes.byref(p))
    n = abi.dspark_workspace_size(ctypes.byref(_with_markov(abi, p, rank=64)))
    R = 2 * 3 * 7
    assert n >= base + R * 4096 * 4 + 2 * R * 64 * 2 + R * 64 * 4
    # a workspace sized without the head is refused for a problem with it
    assert _fwd(abi, p, _params(abi), ws_bytes=base) == abi.DSPARK_ERR_WORKSPACE


def _with_lm_head(abi, p, Ht=256):
    p.target_logits = None
    p.target_hidden = ctypes.c_void_p(0xf0000)
    p.lm_head = ctypes.c_void_p(0x100000)
    p.target_hidden_size = Ht
    return p


def test_teacher_from_hidden_validation_and_workspace(abi):
    prm = _params(abi)
    # FP32 logits are not paired with the tensor-core teacher
    assert _fwd(abi, _with_lm_head(abi, _problem(abi, dtype=abi.DSPARK_F32)), prm) == abi.DSPARK_ERR_UNSUPPORTED
    assert _fwd(abi, _with_lm_head(abi, _problem(abi), Ht=100), prm) == abi.DSPARK_ERR_ALIGNMENT
    p = _with_lm_head(abi, _problem(abi))
    p.lm_head = None
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # teacher logits and teacher hidden states together are ambiguous
    p = _with_lm_head(abi, _problem(abi))
    p.target_logits, p.target_ld = ctypes.c_void_p(0x20000), p.V
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    # the workspace holds the gathered hidden rows and one FP32 chunk of teacher rows
    for B, N, K in ((1, 2, 4), (8, 16, 8)):
        p = _problem(abi, V=4096)
        p.B, p.N, p.K = B, N, K
        base = abi.dspark_workspace_size(ctypes.byref(p))
        n = abi.dspark_workspace_size(ctypes.byref(_with_lm_head(abi, p, Ht=256)))
        R = B * N * K
        assert n >= base + R * 256 * 2 + min(R, 512) * 4096 * 4
        assert n < base + R * 256 * 2 + min(R, 512) * 4096 * 4 + 4096


def test_head_gradient_alignment(abi):
    p = _with_conf_head(abi, _with_markov(abi, _problem(abi)), with_markov=1)
    g = abi.dspark_grads_t()
    g.dlogits, g.dlogits_ld = ctypes.c_void_p(0x70000), p.V
    g.dhidden = ctypes.c_void_p(0x80008)  # not 16-byte aligned
    assert _fwd(abi, p, _params(abi), grads=g) == abi.DSPARK_ERR_ALIGNMENT
    g.dhidden = None
    g.dW2 = ctypes.c_void_p(0x90004)
    assert _fwd(abi, p, _params(abi), grads=g) == abi.DSPARK_ERR_ALIGNMENT


def test_target_norm_validation(abi):
    prm = _params(abi)
    p = _problem(abi)
    p.target_norm_weight = ctypes.c_void_p(0x110000)  # a norm weight without hidden states
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG
    p = _with_lm_head(abi, _problem(abi))
    p.target_norm_weight = ctypes.c_void_p(0x110008)
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_ALIGNMENT
    p.target_norm_weight = ctypes.c_void_p(0x110000)
    p.target_norm_eps = -1.0
    assert _fwd(abi, p, prm) == abi.DSPARK_ERR_INVALID_ARG


def _tp_calls(abi, p, prm, tp, rec=0x200000, ws=0x100000, ws_bytes=1 << 30, grads=None):
    """Status of each of the four vocabulary-parallel calls on the same arguments (the
    head call gets a gradient struct of its own when none is given)."""
    r = ctypes.c_void_p(rec)
    out = abi.dspark_fwd_out_t()
    g4 = grads
    if g4 is None:
        g4 = abi.dspark_grads_t()
        g4.dlogits, g4.dlogits_ld = ctypes.c_void_p(0x70000), p.V
    return (abi.dspark_tp_partials(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), r,
                                   ctypes.c_void_p(ws), ws_bytes, None),
            abi.dspark_tp_l1(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), r, r,
                             ctypes.c_void_p(ws), ws_bytes, None),
            abi.dspark_tp_finish(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), r, ctypes.byref(out),
                                 ctypes.byref(grads) if grads is not None else None, r,
                                 ctypes.c_void_p(ws), ws_bytes, None),
            abi.dspark_tp_heads_bwd(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), r, ctypes.byref(g4),
                                    ctypes.c_void_p(ws), ws_bytes, None))


def test_vocab_parallel_validation(abi):
    """Shard bounds, record buffers, the teacher from hidden states (not taken on this
    path) and the gradient buffers are checked on the host, by every call alike."""
    prm = _params(abi)
    p = _problem(abi, V=1024)
    every = lambda st: (st,) * 4
    # the shard must lie inside the vocabulary
    assert _tp_calls(abi, p, prm, abi.dspark_tp_t(2, 1024, 1024 + 1000)) == every(abi.DSPARK_ERR_INVALID_ARG)
    assert _tp_calls(abi, p, prm, abi.dspark_tp_t(2, -8, 4096)) == every(abi.DSPARK_ERR_INVALID_ARG)
    assert _tp_calls(abi, p, prm, abi.dspark_tp_t(0, 0, 4096)) == every(abi.DSPARK_ERR_INVALID_ARG)
    assert _tp_calls(abi, p, prm, abi.dspark_tp_t(2000, 0, 4096)) == every(abi.DSPARK_ERR_INVALID_ARG)
    assert _tp_calls(abi, p, prm, abi.dspark_tp_t(2, 0, (1 << 30) + 8)) == every(abi.DSPARK_ERR_INVALID_ARG)
    # records: present and 16-byte aligned
    tp = abi.dspark_tp_t(4, 1024, 4096)
    # (without the Markov head the fourth call reads no record and has no work)
    assert _tp_calls(abi, p, prm, tp, rec=0) == (abi.DSPARK_ERR_INVALID_ARG,) * 3 + (abi.DSPARK_OK,)
    assert _tp_calls(abi, p, prm, tp, rec=0x200008) == (abi.DSPARK_ERR_ALIGNMENT,) * 3 + (abi.DSPARK_OK,)
    # the plain problem's rules still hold (shard width under the 16-byte rule, workspace)
    assert _tp_calls(abi, _problem(abi, V=1020), prm, tp) == every(abi.DSPARK_ERR_ALIGNMENT)
    assert _tp_calls(abi, p, prm, tp, ws_bytes=16) == every(abi.DSPARK_ERR_WORKSPACE)
    assert _tp_calls(abi, _problem(abi, target=False), prm, tp) == every(abi.DSPARK_ERR_MISSING_TARGET)
    # the teacher from hidden states on the vocabulary-parallel path keeps every supervised
    # row's teacher shard in the workspace's teacher chunk: more than 512 rows are refused
    # (up to 512 are served; that is tested on the GPU)
    big = _with_lm_head(abi, _problem(abi, target=False))
    big.N, big.K = 65, 8
    assert _tp_calls(abi, big, prm, tp) == every(abi.DSPARK_ERR_UNSUPPORTED)
    # with the Markov head the shard's dE part and the ranks' parts are records too
    pm = _with_markov(abi, _problem(abi))
    g = abi.dspark_grads_t()
    g.dlogits, g.dlogits_ld = ctypes.c_void_p(0x70000), 4096
    assert _tp_calls(abi, pm, prm, tp, rec=0x200008, grads=g) == every(abi.DSPARK_ERR_ALIGNMENT)
    assert _tp_calls(abi, pm, prm, tp, rec=0, grads=g) == every(abi.DSPARK_ERR_INVALID_ARG)
    # a misaligned dlogits stride or head gradient is refused
    g.dlogits_ld = 1028
    assert _tp_calls(abi, p, prm, tp, grads=g)[2:] == (abi.DSPARK_ERR_ALIGNMENT,) * 2
    g.dlogits_ld, g.dW2 = 4096, ctypes.c_void_p(0x80008)
    assert _tp_calls(abi, pm, prm, tp, grads=g)[2:] == (abi.DSPARK_ERR_ALIGNMENT,) * 2
    # NULL params / tp / outputs
    out = abi.dspark_fwd_out_t()
    assert abi.dspark_tp_partials(ctypes.byref(p), None, ctypes.byref(tp), ctypes.c_void_p(0x200000),
                                  ctypes.c_void_p(0x100000), 1 << 30, None) == abi.DSPARK_ERR_INVALID_ARG
    assert abi.dspark_tp_l1(ctypes.byref(p), ctypes.byref(prm), None, ctypes.c_void_p(0x200000),
                            ctypes.c_void_p(0x200000), ctypes.c_void_p(0x100000), 1 << 30,
                            None) == abi.DSPARK_ERR_INVALID_ARG
    assert abi.dspark_tp_finish(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), ctypes.c_void_p(0x200000),
                                None, None, None, ctypes.c_void_p(0x100000), 1 << 30,
                                None) == abi.DSPARK_ERR_INVALID_ARG
    assert abi.dspark_tp_heads_bwd(ctypes.byref(p), ctypes.byref(prm), ctypes.byref(tp), None, None,
                                   ctypes.c_void_p(0x100000), 1 << 30, None) == abi.DSPARK_ERR_INVALID_ARG
    del out


def test_even_shards():
    from speculative_decoding_draft_vocab_b200.torch_api import even_shards
    assert even_shards(151936, 8, 8) == [0, 18992, 37984, 56976, 75968, 94960, 113952, 132944, 151936]
    b = even_shards(50008, 3, 8)
    assert b[0] == 0 and b[-1] == 50008 and all((y - x) % 8 == 0 and y > x for x, y in zip(b, b[1:]))
    assert max(y - x for x, y in zip(b, b[1:])) - min(y - x for x, y in zip(b, b[1:])) <= 8
    with pytest.raises(ValueError):
        even_shards(1001, 2, 8)
    with pytest.raises(ValueError):  # an empty shard
        even_shards(16, 3, 8)
    assert even_shards(24, 3, 8) == [0, 8, 16, 24]


def test_no_alloc_limits_match_header_and_workspace_rule(abi):
    """The fixed scratch of dspark_loss_fwd_noalloc: the header's constants are the
    binding's, and which problems fit follows dspark_workspace_size alone."""
    src = ('#include <stdio.h>\n#include "dspark.h"\n'
           'int main(void) { printf("%d %d\\n", (int)DSPARK_NOALLOC_MAX_ROWS, (int)DSPARK_NOALLOC_BYTES); return 0; }\n')
    with tempfile.TemporaryDirectory() as d:
        with open(os.path.join(d, "n.c"), "w") as f:
            f.write(src)
        subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), os.path.join(d, "n.c"), "-o",
                        os.path.join(d, "n")], check=True)
        rows, nbytes = map(int, subprocess.run([os.path.join(d, "n")], check=True, capture_output=True,
                                               text=True).stdout.split())
    assert (rows, nbytes) == (abi.NOALLOC_MAX_ROWS, abi.NOALLOC_BYTES)
    size = lambda p: abi.dspark_workspace_size(ctypes.byref(p))
    # without heads every micro-batch up to the row limit fits
    p = _problem(abi, V=151936)
    p.B, p.N, p.K = 8, 64, 16
    assert size(p) <= nbytes
    # the Markov head and the teacher from hidden states never fit at a real vocabulary
    assert size(_with_markov(abi, _problem(abi, V=151936), rank=256)) > nbytes
    assert size(_with_lm_head(abi, _problem(abi, V=151936), Ht=4096)) > nbytes
    # a confidence head with hidden size 4096: a few hundred rows fit, the 448-row recipe
    # micro-batch does not
    p = _with_conf_head(abi, _problem(abi, V=151936), H=4096)
    p.B, p.N, p.K = 4, 16, 7
    assert size(p) > nbytes
    p.B, p.N, p.K = 2, 16, 7
    assert size(p) <= nbytes
    # more rows than the limit are refused before any CUDA call
    p = _problem(abi)
    p.B, p.N, p.K = 1, rows // 4 + 1, 4
    out = abi.dspark_fwd_out_t()
    assert abi.dspark_loss_fwd_noalloc(ctypes.byref(p), ctypes.byref(_params(abi)), ctypes.byref(out), None,
                                       None) == abi.DSPARK_ERR_WORKSPACE
