"""The e4m3 softmax branch's numerical method, emulated on the CPU and held
to its tolerance against the fp64 oracle.

Method (the kernel's): q rounded to e4m3 with one scale per (token, head)
row, k and v with one scale per head over video and text tokens (scale =
amax / 448, codes = e4m3(x * 448 / amax), fp32, round to nearest even);
scores q8 . k8 with fp32 accumulation times the row's exponent scale
log2(e) / sqrt(d) * s_q * s_k; the same tiles, lazy running max and exp2
split as the bf16 kernel; P rounded to e4m3 before PV; row sums of the
unrounded P; out = O * s_v / l.

Tolerance (derived here): each code is within 2^-4 of its value, so scores
carry relative errors of a few percent of |q||k| / sqrt(d) and every P and V
element another 2^-4; on the workloads' distributions (q ~ N(0,1), unit keys,
v ~ N(0,1), also the low-rank keys) the emulation lands at rel-L2 0.032 -
0.038 per head. The bound used for o_soft is rel-L2 <= 0.06 and <= 0.08 for
any row. Keys scaled by up to 32x (the max-jump case) make attention sharp
and score errors grow with |k|: the emulation gives about 0.075 there, which
is reported, not held to that bound."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S
from test_exp2_poly import exp2_poly_f32
from test_softmax_algorithm import _max_jump, key_segments

FP8_SOFT_REL_L2 = 0.06
FP8_SOFT_ROW_REL_L2 = 0.08
f32 = np.float32


def e4(x):
    """float32 -> nearest e4m3 value (ties to even), as float32."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).to(
        torch.float32).numpy()


def quant_rows(x):
    amax = np.abs(x).max(axis=-1)
    inv = np.where(amax > 0, f32(448) / np.where(amax > 0, amax, 1), f32(1)).astype(f32)
    sc = np.where(amax > 0, amax / f32(448), f32(1)).astype(f32)
    return e4(x * inv[..., None]), sc


def quant_head(xs):
    amax = f32(max((np.abs(x).max() if x.size else 0.0) for x in xs))
    inv = f32(448) / amax if amax > 0 else f32(1)
    sc = amax / f32(448) if amax > 0 else f32(1)
    return [e4(x * inv) for x in xs], f32(sc)


def emulate_fp8_head(inp, h, threshold=8.0):
    off, F, bf, T, d = inp["off"], inp["F"], inp["block_frames"], inp["T"], inp["d"]
    scale = f32(np.log2(np.e) / np.sqrt(d))
    q8, sq = quant_rows(inp["q"][:, h].astype(f32))
    (k8, kt8), sk = quant_head([inp["k"][:, h].astype(f32), inp["kt"][:, h].astype(f32)])
    (v8, vt8), sv = quant_head([inp["v"][:, h].astype(f32), inp["vt"][:, h].astype(f32)])
    out = np.zeros((inp["N"], d))
    for b in range(O.num_blocks(F, bf)):
        q0, q1 = int(off[bf * b]), int(off[min(bf * b + bf, F)])
        if q1 == q0:
            continue
        Ks, Vs, tiles, base = [], [], [], 0
        for src, a, e in key_segments(off, b, F, bf, T):
            Ks.append((kt8 if src == "t" else k8)[a:e])
            Vs.append((vt8 if src == "t" else v8)[a:e])
            tiles += [(base + i, base + min(i + 128, e - a)) for i in range(0, e - a, 128)]
            base += e - a
        K, V, Q = np.concatenate(Ks), np.concatenate(Vs), q8[q0:q1]
        srow = (scale * sq[q0:q1] * sk).astype(f32)
        m_use, l = None, np.zeros(q1 - q0, f32)
        acc = np.zeros((q1 - q0, d), f32)
        for a, e in tiles:
            s = (Q @ K[a:e].T).astype(f32)
            m_tile = (s.max(axis=1) * srow).astype(f32)
            if m_use is None:
                m_use = m_tile
            else:
                need = m_tile > m_use + f32(threshold)
                fac = np.where(need, np.exp2(np.minimum(m_use - m_tile, 0)), f32(1)).astype(f32)
                m_use = np.where(need, m_tile, m_use)
                l *= fac
                acc *= fac[:, None]
            x = (s * srow[:, None] - m_use[:, None]).astype(f32)
            p = np.exp2(x).astype(f32)
            poly = ((np.arange(e - a) // 2) % 4) == 3
            p[:, poly] = exp2_poly_f32(x[:, poly])
            l += p.sum(axis=1, dtype=f32)
            acc += (e4(p) @ V[a:e]).astype(f32)
        out[q0:q1] = acc * sv / l[:, None]
    return out


def _cases():
    return {
        "mid": S.make_inputs_from(12, [150] * 12, 40, 2, 128, "bf16", seed=0),
        "pages-like": S.make_inputs_from(15, [200] * 15, 64, 2, 128, "bf16", seed=1),
        "hi-res-like": S.make_inputs_from(20, [224] * 20, 64, 2, 128, "bf16", seed=2, k_lowrank=16),
    }


@pytest.mark.parametrize("name", ["mid", "pages-like", "hi-res-like"])
def test_fp8_method_within_derived_tolerance(name):
    inp = _cases()[name]
    for h in range(inp["H"]):
        got = emulate_fp8_head(inp, h)
        ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                    inp["off"], h, inp["block_frames"])
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        row = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert 0.01 < rel <= FP8_SOFT_REL_L2 * 0.75, (name, h, rel)   # really e4m3, with margin
        assert row.max() <= FP8_SOFT_ROW_REL_L2, (name, h, row.max())


def test_fp8_method_on_sharp_attention_is_finite_and_reported():
    # keys scaled by 2^(f // 2): sharp attention, score errors grow with |k|;
    # the method stays finite and within 0.12 there (not the 0.06 bound)
    inp = _max_jump()
    for h in range(inp["H"]):
        got = emulate_fp8_head(inp, h)
        ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                    inp["off"], h, inp["block_frames"])
        assert np.all(np.isfinite(got))
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 0.12
