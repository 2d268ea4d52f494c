"""The design of the bit-exact probe inputs, checked on the CPU (no GPU, no CUDA library).

``tests/test_gpu_index_exact.py`` compares each kernel's output with the oracle's by
``torch.equal``.  That is sound only if (1) the exact result of the definition on the probe
inputs is representable in the dtype, so that any correct kernel produces exactly those bits,
and (2) the inputs would expose a wrong floor, clamp bound or neighbour choice.  (1) is
checked on every probe case; (2) by planting such mistakes in copies of the oracle and
checking that each changes the probe output.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from index_probe import onehot_weight, probe_inputs, shifts_covering
from test_gpu_index_exact import CASES, DT
from test_oracle_mutants import _build_mutant


def _case_inputs(case):
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, near_int) = case
    L_out = oracle.out_length(L, K, s, p, d)
    t = probe_inputs(B, Ci, L, L_out, K, d, og, mask, seed=zlib.crc32(name.encode()) % 1000,
                     near_integer=near_int)
    return {k: (v.to(DT[dt]) if v is not None else None) for k, v in t.items()}


def _weights(case):
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, near_int) = case
    if G == Ci == Co:
        out = []
        for sh in range(K):
            w = torch.zeros(Co, 1, K)
            w[torch.arange(Co), 0, (torch.arange(Co) + sh) % K] = 1.0
            out.append(w)
        return out
    return [onehot_weight(Co, Ci, K, G, sh) for sh in shifts_covering(Co, Ci, K, G)]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_probe_results_are_exact_in_the_dtype(case):
    """Every output of the probe is one sampled value whose exact value the dtype holds."""
    (name, kern, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, near_int) = case
    t = _case_inputs(case)
    ws = _weights(case)
    # the weights read every reduction column (every (channel, tap) pair) at least once
    cover = torch.zeros_like(ws[0][0] if G == Ci == Co else ws[0].sum(0))
    for w in ws:
        cover += w.abs().sum(0) if not (G == Ci == Co) else w.abs().sum(0)
    assert bool((cover > 0).all()), name
    for w in ws:
        r = oracle.forward(t["x"], t["offsets"], t["mask"], w.to(DT[dt]), None, s, p, d, G, og,
                           unc)
        if near_int and dt == "f32":
            # one rounding of the exact value to fp32: the oracle's double is that value
            continue
        back = torch.from_numpy(np.ascontiguousarray(r)).to(DT[dt]).double().numpy()
        assert np.array_equal(back, r), name


# Index mistakes a kernel could make, planted in copies of the oracle: each must change the
# output on the probe inputs.
INDEX_MUTANTS = [
    ("floor one too small", "*i0 = (int64_t)fl;", "*i0 = (int64_t)fl - 1;"),
    ("nearest instead of floor", "float fl = floorf(pos);", "float fl = rintf(pos);"),
    ("trunc instead of floor", "float fl = floorf(pos);", "float fl = truncf(pos);"),
    ("upper clamp one past the field", "float hi = (float)(start + S->dilation * (S->K - 1));",
     "float hi = (float)(start + S->dilation * (S->K - 1) + 1);"),
    ("lower clamp one before the field", "float lo = (float)start;",
     "float lo = (float)(start - 1);"),
    ("neighbours one to the right",
     "double v = (1.0 - (double)f) * x_at(x, S, b, ci, i0) + (double)f * x_at(x, S, b, ci, i0 + 1);",
     "double v = (1.0 - (double)f) * x_at(x, S, b, ci, i0 + 1) + (double)f * x_at(x, S, b, ci, i0 + 2);"),
    ("fraction dropped", "*f = pos - (float)(*i0);", "*f = 0.0f;"),
]


def _probe_for(name):
    case = next(c for c in CASES if c[0] == name)
    return case, _case_inputs(case), _weights(case)


@pytest.mark.parametrize("name,old,new", INDEX_MUTANTS, ids=[m[0] for m in INDEX_MUTANTS])
def test_probe_catches_index_mistakes(tmp_path, name, old, new):
    mut = _build_mutant(str(tmp_path), old, new)
    # a constrained case (clamp bounds) and an unconstrained one (far and window-crossing
    # offsets); a mutant must change at least one output bit of the dtype in one of them
    caught = []
    for cname in ("tc_k5_mask_og4_constrained", "tc_k9_strided_groups_unconstrained"):
        case, t, ws = _probe_for(cname)
        (_, _, dt, B, Ci, Co, K, L, s, p, d, G, og, mask, unc, _) = case
        for w in ws:
            a = [o.forward(t["x"], t["offsets"], t["mask"], w.to(DT[dt]), None, s, p, d, G, og,
                           unc) for o in (oracle.get(), mut)]
            ra, rb = (torch.from_numpy(np.ascontiguousarray(v)).to(DT[dt]) for v in a)
            if not torch.equal(ra, rb):
                caught.append(cname)
                break
    assert caught, f"the probe inputs do not expose: {name}"
    if "clamp" not in name:
        # mistakes in the floor or the neighbours show in both modes
        assert len(caught) == 2, (name, caught)
