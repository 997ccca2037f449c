"""Error budget of the decode kernel's int8 P.V arithmetic, on the CPU.

For ternary pages at GQA <= 4 the kernel forms P.V from P quantised to
unsigned fixed point: in a full entry of 8 pages, P = 2^(s - m_e) *
gamma_v / gamma_max <= 1 in steps of 2^-15 (two 8-bit digits), m_e the
entry's own score maximum per head; the digit sums are exact (int32) and
are folded into floating point once per entry, scaled by 2^(m_e - m) with m
the running maximum; the normaliser sums P unrounded.  The GPU parity tests
compare the kernel with the fp64 oracle on reduced sizes in full and on a
few sampled sequences at full size.  This test replays that quantisation
step alone (exact scores, exact decoded values) for whole
Llama-3-8B-shaped sequences of 32768 tokens, for scores whose maximum keeps
moving and for sharper softmaxes (scores x2 .. x8), and checks the error
against the fp64 softmax stays well inside the attention bar (relative L2
1e-3).  It also records why the digits are taken per entry: relative to
the running maximum instead, a softmax sharpened x4 loses ~9.6e-4, since
its many mid-weight tokens get few bits.  It models the arithmetic, not
the kernel's code."""

import math

import numpy as np
import pytest

import oracle as O
import synth
from kvc_testlib import bits

STEP = 2.0 ** -15


def _ternary_values(pages_bits):
    """bf16 pages [n][P][D] (one KV head) -> exact decoded values [n*P][D]
    and the per-page gamma, through the oracle's codec."""
    n, p, d = pages_bits.shape
    codes, gamma = O.quantize_pack_ternary(pages_bits[:, None])
    vals = np.stack([O.ternary_decoded_f64(codes[i, 0], gamma[i, 0]) for i in range(n)])
    return vals.reshape(n * p, d), gamma[:, 0].astype(np.float64)


def _model_output(s_log2, v_codes, v_gamma_page, per_entry=True, entry_pages=8, page=16):
    """softmax(s) . V with P in 2^-15 fixed point folded per entry of 8
    pages, s in log2 units, V = gamma_page * codes; the digits relative to
    each entry's own maximum (the kernel), or with per_entry False relative
    to the running maximum.  Returns the output row."""
    n_tok, d = v_codes.shape
    n_pages = n_tok // page
    m = -math.inf
    acc = np.zeros(d)
    l_sum = 0.0
    for e0 in range(0, n_pages, entry_pages):
        e1 = min(n_pages, e0 + entry_pages)
        t0, t1 = e0 * page, e1 * page
        s = s_log2[t0:t1]
        r = float(s.max())
        if r > m:                                    # the running maximum moves
            m_new = math.ceil(r) if m == -math.inf else m + math.ceil(r - m)
            a = 0.0 if m == -math.inf else 2.0 ** (m - m_new)
            acc *= a
            l_sum *= a
            m = m_new
        m_e = r if per_entry else m
        scale = 2.0 ** (m_e - m)                     # <= 1
        p = np.exp2(s - m_e)                         # <= 1
        l_sum += float(p.sum()) * scale
        g_page = np.repeat(v_gamma_page[e0:e1], page)
        gmax = float(g_page.max())
        digits = np.rint(p * g_page / gmax / STEP)   # two exact 8-bit digits: 0 .. 2^15
        assert digits.max() <= 2 ** 15
        # exact integer sums of digits x codes, folded once per entry
        acc += gmax * STEP * scale * (digits[:, None] * v_codes[t0:t1]).sum(axis=0)
    return acc / l_sum


def _reference(s_log2, v_vals):
    w = np.exp2(s_log2 - s_log2.max())
    return (w[:, None] * v_vals).sum(axis=0) / w.sum()


def _rel(out, ref):
    return float(np.linalg.norm(out - ref) / np.linalg.norm(ref))


def _sequence():
    inp = synth.make_decode_inputs("llama8b", seed=1, batch=1, n_q_heads=4, n_kv_heads=1)
    d = inp["cfg"]["head_dim"]
    q = inp["q"].float().numpy().astype(np.float64)[0]               # [4][D]
    k_vals, _ = _ternary_values(bits(inp["k_pages"][0, :, 0]))         # [32768][D]
    v_vals, v_gamma = _ternary_values(bits(inp["v_pages"][0, :, 0]))
    v_codes = v_vals / np.repeat(v_gamma, 16)[:, None]                 # exact codes in {-1, 0, 1}
    return q, k_vals, v_vals, v_codes, v_gamma, math.log2(math.e) / math.sqrt(d)


def _worst(pattern, per_entry):
    q, k_vals, v_vals, v_codes, v_gamma, scale_log2 = _sequence()
    worst = 0.0
    for h in range(q.shape[0]):
        s = (k_vals @ q[h]) * scale_log2
        if pattern == "rising":          # the maximum moves on almost every page
            s = s + np.linspace(0.0, 40.0, s.size)
        elif pattern.startswith("sharp"):  # a few dominant tokens, a long tail of mid weights
            s = float(pattern[5:]) * s
        out = _model_output(s, v_codes, v_gamma, per_entry)
        worst = max(worst, _rel(out, _reference(s, v_vals)))
    return worst


@pytest.mark.parametrize("pattern", ["workload", "rising", "sharp2", "sharp4", "sharp8"])
def test_fixed_point_p_error_is_far_inside_the_bar(pattern):
    # the kernel's arithmetic: digits relative to each entry's own maximum
    worst = _worst(pattern, per_entry=True)
    assert worst < 2.5e-4, worst


def test_running_maximum_digits_lose_bits_on_sharper_softmax():
    # the reason the digits are taken per entry
    running = _worst("sharp4", per_entry=False)
    assert running > 4 * _worst("sharp4", per_entry=True)
    assert running < 1e-3
