"""Full-size parity of the paths the bench times, group by group, against the
oracle (H-Scale summary, sec. 3 "Group-wise scale selection"; ScaleSweep
summary, sec. 3):

  * Llama-3-8B-shaped projections and the Llama-3.3-70B-shaped MLP through
    nvfp4_quantize_layer (one call per layer, reductions streamed beside the
    sweeps);
  * the 128-expert mixture-of-experts layer through
    nvfp4_quantize_grouped_layer.

Every h column is compared with the oracle's sum of squares (1e-5 relative),
every S bit for bit, and every group of every matrix with the oracle's sweep
fed the GPU's h (at least 99.99% of groups byte-equal; every other group's
exact loss within 1e-6 relative of the oracle's).  The end-to-end mismatch
rate, each side using its own h, is reported beside it.  The figures are
printed in the run's summary.  Needs a B200 and a few minutes of host time."""
import numpy as np
import pytest
import torch

from parity import assert_parity, check_h, compare_groups, matrix_groups, to_bits

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"


@pytest.fixture(scope="module")
def nv():
    import block_scale_search_b200 as nv
    nv.lib()
    return nv


def _check_matrix(orc, report, name, W, h_gpu, h_ref, S_dev, q_max, codes, scales, lo, hi):
    """S, then every group against the oracle with the GPU's h (asserted) and
    with the oracle's own h (reported)."""
    bits = to_bits(W)
    S_ref, amax_ref, st = orc.global_scale(bits, q_max)
    S = np.float32(S_dev.item())
    assert st == 0 and S == S_ref, f"{name}: S {S} vs oracle {S_ref}"
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    rc, rs, _ = orc.parallel_sweep_quantize(bits, h_gpu, float(S), lo, hi)
    w, hh, _, _ = matrix_groups(bits, gc, gs, h_gpu)
    res = compare_groups(orc, w, hh, float(S), gc, gs, rc, rs)
    # end to end: the oracle's sweep on the oracle's own h
    if h_ref is not None and not np.array_equal(h_ref.view(np.uint32), h_gpu.view(np.uint32)):
        ec, es, _ = orc.parallel_sweep_quantize(bits, h_ref, float(S), lo, hi)
        e2e = (es.reshape(-1) == gs.reshape(-1)) & np.all(
            ec.reshape(-1, 8) == gc.reshape(-1, 8), axis=1)
        e2e_mis = int((~e2e).sum())
    else:
        e2e_mis = res["mismatch"]
    report(f"{name}: {res['groups']} groups, same-h mismatches {res['mismatch']} "
           f"(worst rel loss {res['worst_rel_loss']:.2e}), own-h mismatches {e2e_mis} "
           f"({e2e_mis / res['groups']:.2e})")
    assert_parity(res, name)
    return res, e2e_mis


def _layer(orc, nv, report, wl):
    keys = list(wl.calibs)
    Xs = [wl.calibs[k].make(DEV) for k in keys]
    Ws = [m.make(DEV) for m in wl.matrices]
    inputs = [keys.index(m.x_key) for m in wl.matrices]
    outs, hs = nv.quantize_layer_many(Ws, Xs, inputs, wl.q_max, -9, 6)
    torch.cuda.synchronize()
    h_gpu, h_ref = [], []
    for k, X, h in zip(keys, Xs, hs):
        hg = h.cpu().numpy()
        hr = orc.parallel_diag_hessian(X.cpu())
        worst = check_h(hg, hr)
        report(f"{wl.name}.h[{k}]: {hg.size} columns, worst rel error {worst:.2e}")
        h_gpu.append(hg)
        h_ref.append(hr)
    del Xs
    torch.cuda.empty_cache()
    for m, W, k, (codes, scales, S, _, status) in zip(wl.matrices, Ws, inputs, outs):
        assert status.item() == 0
        _check_matrix(orc, report, f"{wl.name}.{m.name}", W, h_gpu[k], h_ref[k], S, wl.q_max,
                      codes, scales, -9, 6)


def test_llama3_8b_projections_full(orc, nv, parity_report):
    import workloads
    _layer(orc, nv, parity_report, workloads.llama3_8b())
    torch.cuda.empty_cache()


def test_llama33_70b_mlp_full(orc, nv, parity_report):
    import workloads
    _layer(orc, nv, parity_report, workloads.llama33_70b_mlp())
    torch.cuda.empty_cache()


def test_moe_grouped_layer_full(orc, nv, parity_report):
    import workloads
    wl = workloads.moe_grouped(device=DEV)
    offs = wl.calibs["gu"].row_offsets
    off_d = torch.as_tensor(offs, dtype=torch.int64, device=DEV)
    X1 = wl.calibs["gu"].make(DEV)
    X2 = wl.calibs["down"].make(DEV)
    first = [m for m in wl.matrices if m.x_key == "gu"]
    second = [m for m in wl.matrices if m.x_key == "down"]
    W1 = [m.make(DEV) for m in first]
    W2 = [m.make(DEV) for m in second]
    o1, o2, h1, h2, S, _, status = nv.quantize_grouped_layer(
        list(zip(W1, [m.expert for m in first])), list(zip(W2, [m.expert for m in second])),
        X1, X2, off_d, wl.q_max, -9, 6)
    torch.cuda.synchronize()
    assert int(status.abs().max().item()) == 0
    h_gpu = {"gu": h1.cpu().numpy(), "down": h2.cpu().numpy()}
    h_ref = {k: np.zeros_like(v) for k, v in h_gpu.items()}
    for k, X in (("gu", X1), ("down", X2)):
        for e in range(wl.experts):
            h_ref[k][e] = orc.parallel_diag_hessian(X[offs[e]:offs[e + 1]].cpu())
        worst = check_h(h_gpu[k], h_ref[k])
        parity_report(f"{wl.name}.h[{k}]: {wl.experts} experts x {h_gpu[k].shape[1]} columns, "
                      f"worst rel error {worst:.2e}")
    del X1, X2
    torch.cuda.empty_cache()
    total = {"groups": 0, "same": 0, "own": 0}
    n1 = len(first)
    for i, (m, W, (codes, scales, _)) in enumerate(zip(first + second, W1 + W2, o1 + o2)):
        hg, hr = h_gpu[m.x_key][m.expert], h_ref[m.x_key][m.expert]
        res, own = _check_matrix(orc, lambda s: None, m.name, W, hg, hr, S[i], wl.q_max, codes,
                                 scales, -9, 6)
        total["groups"] += res["groups"]
        total["same"] += res["mismatch"]
        total["own"] += own
    parity_report(f"{wl.name}: {len(first) + len(second)} matrices, {total['groups']} groups, "
                  f"same-h mismatches {total['same']} (each matrix within 99.99% and 1e-6), "
                  f"own-h mismatches {total['own']} ({total['own'] / total['groups']:.2e})")
    assert n1 == 2 * wl.experts
