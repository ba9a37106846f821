"""Full-size parity of the CUDA path against the CPU oracle.

The prefill-shaped layer (T = 8192) and the 24-layer stack (T = 2048, skewed
routing) run on the GPU exactly as bench.py runs them: one context sized for
the workload's T, one moe_forward per layer.  The oracle is too slow for every
token of these workloads, so it checks a seeded sample of rows (the first, the
last and random ones); each row of the block depends only on its own token, so
a sampled row is checked against exactly what the oracle computes for it.
Properties that hold at any size are checked on every row.

Stack parity is teacher-forced: the oracle's layer l gets the GPU's layer
l - 1 output for the sampled rows.  The drift of a few rows carried through all
24 layers by the oracle alone is checked against a loose bound and reported.
The stack amplifies small differences: the oracle chain itself, with a
Gaussian perturbation of mean relative size 1.5e-3 added to every layer's
output (the size of the GPU path's per-layer difference), ends 2.4e-2 to
5.7e-2 (mean relative) away from the unperturbed chain after 24 layers, and
2e-2 to 2.8e-2 with 0.5e-3 per layer.  The bound on the GPU's drift is 0.1.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import sparse_moe_rmsnorm_b200 as moe
from moe_inputs import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_config_inputs, make_tokens
from _parity import GAP, compare_block

pytestmark = pytest.mark.gpu

# the fp32 accumulator (before the bf16 output cast): these batches reach the tensor core with two
# E4M3 terms per activation (about bf16's 8 bits); as in test_gpu_parity, the bound asks for at least
# the exactness of bf16 operands, which give 2.9e-3 on a 2880-wide layer
ACC_MEAN_REL = 2.5e-3
# end-to-end drift of the 24-layer stack (see the module docstring for the calibration)
DRIFT_MEAN_REL = 0.1


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _sample_rows(T, n, seed):
    rng = np.random.default_rng(seed)
    rest = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return np.array(sorted({0, T - 1, *rest.tolist()}))


def _acc_rows(m, x_bits_rows, rows, k, T):
    """x + the token's weighted expert rows, summed in float64, for the sampled rows only."""
    pair_row = m.workspace("pair_row", T).view(T, k)[torch.from_numpy(rows).cuda()]
    orows = m.workspace("out_rows", T)[pair_row.view(-1).long()].view(len(rows), k, -1)
    return bf16_bits_to_f32(x_bits_rows).astype(np.float64) + orows.double().sum(dim=1).cpu().numpy()


def _check_rows(m, y, idx, wts, x_bits_rows, rows, inp, cfg, label):
    ref = oracle.moe_forward(inp, cfg.k, cfg.eps, x=x_bits_rows)
    y_rows = y[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    res = compare_block(y_rows, idx[rows], wts[rows], ref, cfg.k, cfg.E)
    acc = compare_block(_acc_rows(m, x_bits_rows, rows, cfg.k, cfg.T), idx[rows], wts[rows], ref, cfg.k, cfg.E)
    print(label, res, "| fp32 accumulator:", {k_: acc[k_] for k_ in ("max_rel", "mean_rel")})
    assert res["ok"], (label, res)
    assert res["w_max_err"] < 1e-5, (label, res)
    assert acc["mean_rel"] <= ACC_MEAN_REL, (label, acc)
    return ref


def _check_every_row(m, y, idx, cfg):
    """Properties of the whole batch: finite output, k distinct experts in range per token, and the
    grouping accounts for every (token, expert) pair."""
    assert torch.isfinite(y.float()).all()
    assert np.all((idx >= 0) & (idx < cfg.E))
    srt = np.sort(idx, axis=1)
    assert np.all(srt[:, 1:] != srt[:, :-1]), "a token chose an expert twice"
    counts = m.workspace("counts", cfg.T).cpu().numpy()
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=cfg.E))
    return counts


def test_prefill20b_sampled_rows():
    cfg = CONFIGS["prefill20b"]
    inp = make_config_inputs(cfg)
    w = moe.MoEWeights.from_numpy(inp)
    x = _bf16_dev(inp["x"])
    m = moe.MoE(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps)
    y, idx, wts = m.forward(x, w, routing=True)
    torch.cuda.synchronize()
    assert m.sync_status() == moe.MOE_OK
    idx = idx.cpu().numpy()
    wts = wts.cpu().numpy().astype(np.float64)
    counts = _check_every_row(m, y, idx, cfg)
    print("prefill20b expert load max/mean %.2f" % (counts.max() / counts.mean()))
    rows = _sample_rows(cfg.T, 48, seed=11)
    _check_rows(m, y, idx, wts, inp["x"][rows], rows, inp, cfg, "prefill20b")
    m.close()


def test_stack20b_teacher_forced_sampled_rows():
    cfg = CONFIGS["stack20b"]
    x0 = make_tokens(np.random.Generator(np.random.PCG64(cfg.seed)), cfg.T, cfg.d)
    m = moe.MoE(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps)
    rows = _sample_rows(cfg.T, 8, seed=12)
    chain_rows = rows[:2]
    x_chain = x0[chain_rows]                 # carried through the layers by the oracle alone
    chain_near_tie = np.zeros(len(chain_rows), dtype=bool)
    x = _bf16_dev(x0)
    skew = []
    for layer in range(cfg.layers):
        inp = make_config_inputs(cfg, layer)
        w = moe.MoEWeights.from_numpy(inp)
        y, idx, wts = m.forward(x, w, routing=True)
        torch.cuda.synchronize()
        assert m.sync_status() == moe.MOE_OK
        idx = idx.cpu().numpy()
        wts = wts.cpu().numpy().astype(np.float64)
        counts = _check_every_row(m, y, idx, cfg)
        skew.append(counts.max() / counts.mean())
        x_rows = _bits(x[torch.from_numpy(rows).cuda()])
        _check_rows(m, y, idx, wts, x_rows, rows, inp, cfg, "stack layer %d" % layer)
        ref_c = oracle.moe_forward(inp, cfg.k, cfg.eps, x=x_chain)
        s = -np.sort(-ref_c["logits"].astype(np.float64), axis=1)
        chain_near_tie |= (s[:, cfg.k - 1] - s[:, cfg.k]) < GAP
        x_chain = f32_to_bf16_bits(ref_c["y"].astype(np.float32))
        x = y
        del w
    print("stack expert load max/mean per layer:", ["%.1f" % v for v in skew])
    y_gpu = bf16_bits_to_f32(_bits(x[torch.from_numpy(chain_rows).cuda()])).astype(np.float64)
    y_ora = bf16_bits_to_f32(x_chain).astype(np.float64)
    for i in range(len(chain_rows)):
        diff = np.abs(y_gpu[i] - y_ora[i])
        rel = diff.sum() / np.abs(y_ora[i]).sum()
        print("24-layer drift, row %d: mean rel %.3g, max rel %.3g%s" % (
            chain_rows[i], rel, diff.max() / np.abs(y_ora[i]).max(),
            " (a near tie on the way: not asserted)" if chain_near_tie[i] else ""))
        if not chain_near_tie[i]:
            assert rel <= DRIFT_MEAN_REL
    m.close()
