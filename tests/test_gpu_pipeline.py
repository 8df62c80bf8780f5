"""Layer orchestration on the GPU against the CPU oracle.

* LayerStreamer: layers streamed from pinned host memory through a 2-slot
  device ring on three streams give, layer by layer, exactly the oracle's
  results (a slot reused too early would mix two layers' data).
* One full layer of the 36-layer Qwen3-8B-shaped stack (2048 tokens per
  layer, 7 linears in 4 search groups) through GroupJob, every group
  compared with the oracle: bit-exact means, scales, codes, words, index;
  error sums within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from post_int4_weight_b200 import pipeline
from post_int4_weight_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-5
TIE_RTOL = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"


def _oracle_group(Ws, X, g, n_grid, output_mode):
    x = oracle.act_stats(X)
    if output_mode:
        err = oracle.output_error(X, Ws[0], x, g, n_grid)
        best = int(np.argmin(err))
        s = oracle.scale_table(x, n_grid)[best]
    else:
        err, best, s = oracle.scale_search(Ws, x, g, n_grid)
    packs = [oracle.quantize_pack(W, s, g, 8) for W in Ws]
    return x, err, best, s, packs


def _compare(got, Ws, X, g, n_grid, output_mode):
    """got = (x or None, err, best, s_best, packs) as numpy."""
    x_o, err_o, best_o, s_o, packs_o = _oracle_group(Ws, X, g, n_grid, output_mode)
    x, err, best, s, packs = got
    if x is not None:
        assert np.array_equal(x, x_o)
    np.testing.assert_allclose(err, err_o, rtol=ERR_RTOL, atol=0)
    if best != best_o:
        assert abs(err_o[best] - err_o[best_o]) <= TIE_RTOL * err_o[best_o]
        return
    assert np.array_equal(s, s_o)
    for (qw, sc, qz), (qw_o, sc_o, qz_o) in zip(packs, packs_o):
        assert np.array_equal(qw, qw_o)
        assert np.array_equal(sc.view(np.uint16), sc_o.view(np.uint16))
        assert np.array_equal(qz, qz_o)


def _small_layer(seed):
    """Two search groups: (256 + 128) x 512 with 64 tokens, 128 x 1024 with
    96 tokens."""
    return [([wl.weight(256, 512, seed + 1), wl.weight(128, 512, seed + 2)],
             wl.activations(64, 512, seed)),
            ([wl.weight(128, 1024, seed + 4)], wl.activations(96, 1024, seed + 3))]


@pytest.mark.parametrize("output_mode", [False, True])
def test_layer_streamer_matches_oracle_per_layer(output_mode):
    g, n_grid, n_layers = 128, 20, 5
    layers = [_small_layer(1000 + 10 * l) for l in range(n_layers)]
    if output_mode:
        layers = [[(Ws[:1], X) for Ws, X in lay] for lay in layers]
    host = [[([W.pin_memory() for W in Ws], X.pin_memory()) for Ws, X in lay]
            for lay in layers]
    st = pipeline.LayerStreamer(layers[0], "cuda", g, n_grid, output_mode)
    out = [st.host_outputs() for _ in range(n_layers)]
    st.run(host, out)
    torch.cuda.synchronize()
    for lay, res in zip(layers, out):
        for (Ws, X), (err, best, s, packs) in zip(lay, res):
            got = (None, err.numpy(), int(best[0]), s.numpy(),
                   [tuple(t.numpy() for t in pk) for pk in packs])
            _compare(got, [W.numpy() for W in Ws], X.numpy(), g, n_grid, output_mode)


def test_stack36_layer_full_parity():
    work = wl.WORKLOADS["qwen3_8b_stack36"]
    layer = work.layers - 1
    groups = wl.group_inputs(work, layer)
    dev = torch.device("cuda")
    jobs = [pipeline.GroupJob([W.to(dev) for W in Ws], X.to(dev), 128, work.n_grid)
            for _, Ws, X in groups]
    wss = pipeline.Workspaces(jobs, dev)
    for j in jobs:
        j.run(wss)
    torch.cuda.synchronize()
    for (grp, Ws, X), j in zip(groups, jobs):
        got = (j.x.cpu().numpy(), j.err.cpu().numpy(), int(j.best.cpu()[0]),
               j.s_best.cpu().numpy(), [tuple(t.cpu().numpy() for t in pk) for pk in j.packs])
        _compare(got, [W.numpy() for W in Ws], X.numpy(), 128, work.n_grid, False)


def test_layer_streamer_with_clip_search():
    """Three layers streamed with the clip search on: for every member the
    clip indices agree with the oracle at the chosen scale (ties within 1e-6
    exempt) and the packed output equals the oracle's pack of those indices."""
    g, n_grid, n_clip = 128, 20, 10
    layers = [_small_layer(2000 + 10 * l) for l in range(3)]
    host = [[([W.pin_memory() for W in Ws], X.pin_memory()) for Ws, X in lay]
            for lay in layers]
    st = pipeline.LayerStreamer(layers[0], "cuda", g, n_grid, False, n_clip=n_clip)
    out = [st.host_outputs() for _ in range(3)]
    st.run(host, out)
    torch.cuda.synchronize()
    for lay, res in zip(layers, out):
        for (Ws, X), (err, best, s, packs) in zip(lay, res):
            x = oracle.act_stats(X.numpy())
            err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x, g, n_grid)
            assert int(best[0]) == best_o
            assert np.array_equal(s.numpy(), s_o)
            for W, pk in zip(Ws, packs):
                qw, sc, qz, idx = (t.numpy() for t in pk)
                idx_o, _ = oracle.clip_search(W.numpy(), x, s_o, g, n_clip)
                Wf = W.numpy().astype(np.float32)
                for r, k in np.argwhere(idx != idx_o):
                    sl = slice(k * g, (k + 1) * g)
                    e1 = oracle.clip_group_error(Wf[r, sl], s_o[sl], x[sl],
                                                 oracle.clip_ratio(idx[r, k]))
                    e2 = oracle.clip_group_error(Wf[r, sl], s_o[sl], x[sl],
                                                 oracle.clip_ratio(idx_o[r, k]))
                    assert abs(e1 - e2) <= TIE_RTOL * e2
                qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s_o, g, 8, idx)
                assert np.array_equal(qw, qw_o)
                assert np.array_equal(sc.view(np.uint16), sc_o.view(np.uint16))
                assert np.array_equal(qz, qz_o)


def test_layer_streamer_with_output_clip():
    """Two layers streamed with the clip search scored on the output: for
    every member the indices agree with the oracle's output-space clip at the
    chosen scale (a differing index only where the two ratios' output scores
    tie within 1e-5) and the packed output equals the oracle's pack of the
    GPU's indices."""
    g, n_grid, n_clip = 128, 20, 10
    layers = [_small_layer(3000 + 10 * l) for l in range(2)]
    host = [[([W.pin_memory() for W in Ws], X.pin_memory()) for Ws, X in lay]
            for lay in layers]
    st = pipeline.LayerStreamer(layers[0], "cuda", g, n_grid, False, n_clip=n_clip,
                                clip_space="output")
    out = [st.host_outputs() for _ in range(2)]
    st.run(host, out)
    torch.cuda.synchronize()
    for lay, res in zip(layers, out):
        for (Ws, X), (err, best, s, packs) in zip(lay, res):
            Xn = X.numpy()
            x = oracle.act_stats(Xn)
            err_o, best_o, s_o = oracle.scale_search([W.numpy() for W in Ws], x, g, n_grid)
            assert int(best[0]) == best_o
            assert np.array_equal(s.numpy(), s_o)
            Xd = Xn.astype(np.float64)
            for W, pk in zip(Ws, packs):
                qw, sc, qz, idx = (t.numpy() for t in pk)
                idx_o, _ = oracle.clip_search_output(Xn, W.numpy(), s_o, g, n_clip)
                diff = np.argwhere(idx != idx_o)
                assert len(diff) <= max(2, idx_o.size // 1000)
                for r, k in diff:
                    cols = slice(k * g, (k + 1) * g)
                    w = W.numpy()[r].astype(np.float32)

                    def score(i):
                        q, qs = oracle.fake_quant_group_clip(w[cols], s_o[cols],
                                                             oracle.clip_ratio(int(i)))
                        dw = (w[cols].astype(np.float64)
                              - q.astype(np.float64) * qs / s_o[cols].astype(np.float64))
                        y = Xd[:, cols] @ dw
                        return float(y @ y)
                    a, b = score(idx[r, k]), score(idx_o[r, k])
                    assert abs(a - b) <= 1e-5 * b
                qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s_o, g, 8, idx)
                assert np.array_equal(qw, qw_o)
                assert np.array_equal(sc.view(np.uint16), sc_o.view(np.uint16))
                assert np.array_equal(qz, qz_o)


def test_norm_group_geomean_kernel_bit_exact():
    from post_int4_weight_b200 import awq
    rng = np.random.default_rng(61)
    for n in (1, 2, 3, 5, 8):
        ss = [np.exp(rng.standard_normal(4096) * 3).astype(np.float32) for _ in range(n)]
        ss[0][:4] = [1e-30, 1e30, 1.0, 3.0e-8]          # extremes of the fp32 range
        g = awq.norm_group_scale([torch.from_numpy(x).cuda() for x in ss])
        torch.cuda.synchronize()
        assert np.array_equal(g.cpu().numpy(), oracle.geomean_scales(ss)), n


def test_norm_group_mode_qkv_block_group():
    """The Qwen3-8B q/k/v group (4096 + 1024 + 1024 rows x 4096, 16384 tokens)
    in geomean mode: per-member searches, the shared scale and the three
    re-quantised linears against the oracle."""
    work = wl.WORKLOADS["qwen3_8b_block"]
    grp, Ws, X = wl.group_inputs(work)[0]
    dev = torch.device("cuda")
    job = pipeline.GroupJob([W.to(dev) for W in Ws], X.to(dev), 128, 20, scale_mode="geomean")
    job.run(pipeline.Workspaces([job], dev))
    torch.cuda.synchronize()
    x = oracle.act_stats(X.numpy())
    assert np.array_equal(job.x.cpu().numpy(), x)
    ss = []
    for m, W in enumerate(Ws):
        err_o, best_o, s_o = oracle.scale_search([W.numpy()], x, 128, 20)
        np.testing.assert_allclose(job.err[m, :20].cpu().numpy(), err_o, rtol=ERR_RTOL, atol=0)
        b = int(job.best[m, 0].cpu())
        if b != best_o:
            assert abs(err_o[b] - err_o[best_o]) <= TIE_RTOL * err_o[best_o]
            s_o = oracle.scale_table(x, 20)[b]        # follow the GPU's tie choice
        assert np.array_equal(job.member_s[m].cpu().numpy(), s_o)
        ss.append(s_o)
    s_shared = oracle.geomean_scales(ss)
    assert np.array_equal(job.s_best.cpu().numpy(), s_shared)
    for W, pk in zip(Ws, job.packs):
        qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s_shared, 128, 8)
        assert np.array_equal(pk[0].cpu().numpy(), qw_o)
        assert np.array_equal(pk[1].cpu().numpy().view(np.uint16), sc_o.view(np.uint16))
        assert np.array_equal(pk[2].cpu().numpy(), qz_o)


def test_checkpointed_layers_resume_bit_identical(tmp_path):
    """Three small layers quantised through the library with a checkpoint;
    the first pass stops after layer 0 (a host-side stop, as a preempted job
    would), the rerun computes only layers 1 and 2, and every layer's packed
    output equals an uninterrupted run's bit for bit; layer 1 also equals
    the oracle."""
    from post_int4_weight_b200 import checkpoint as ck
    dev = torch.device("cuda")
    cfg = {"d_out": 256, "d_in": 512, "T": 64, "g": 128, "n_grid": 20}

    def inputs(l):
        return wl.weight(256, 512, 500 + l), wl.activations(64, 512, 600 + l)

    def compute_fn(stop_at=None, calls=None):
        def f(l):
            if calls is not None:
                calls.append(l)
            if l == stop_at:
                raise RuntimeError("stop")
            W, X = inputs(l)
            job = pipeline.GroupJob([W.to(dev)], X.to(dev), 128, 20)
            wss = pipeline.Workspaces([job], dev)
            job.run(wss)
            qw, sc, qz = job.packs[0]
            return {"qweight": qw, "scales": sc, "qzeros": qz, "s_best": job.s_best,
                    "best": job.best}
        return f

    c = ck.StackCheckpoint(str(tmp_path / "a"), cfg)
    with pytest.raises(RuntimeError):
        ck.run_layers(range(3), compute_fn(stop_at=1), c)
    calls = []
    out = ck.run_layers(range(3), compute_fn(calls=calls), ck.StackCheckpoint(str(tmp_path / "a"), cfg))
    assert calls == [1, 2]
    ref = ck.run_layers(range(3), compute_fn(), ck.StackCheckpoint(str(tmp_path / "b"), cfg))
    for l in range(3):
        for k in out[l]:
            assert torch.equal(out[l][k], ref[l][k]), (l, k)
    W, X = inputs(1)
    x = oracle.act_stats(X.numpy())
    _, best_o, s_o = oracle.scale_search([W.numpy()], x, 128, 20)
    qw_o, sc_o, qz_o = oracle.quantize_pack(W.numpy(), s_o, 128, 8)
    assert int(out[1]["best"][0]) == best_o
    assert np.array_equal(out[1]["qweight"].numpy(), qw_o)
    assert np.array_equal(out[1]["scales"].numpy().view(np.uint16), sc_o.view(np.uint16))
