"""The 48-block residual chain of the Keras-default shape at full size (D=2048, E=60, k=4,
I=1408, T=4096): x_{l+1} = x_l + MoE_l(x_l), every block with its own seeded weights.

Rows are independent through the whole chain (a token's output depends only on its own
input), so the oracle follows a subset of rows while the GPU runs the whole batch:

* Teacher forcing, every layer.  The GPU's batch at layer l is its own free-running state
  with the tracked rows R replaced by the oracle's bf16 trajectory.  The GPU output of R,
  and of sampled rows at the edges of this layer's expert tiles (whatever the GPU's own
  state holds there), is checked against the oracle run on exactly the same inputs:
  routing exact on decisive tokens and valid elsewhere, selection from the GPU's own logits
  bit-exact for all 4096 tokens, and the output criterion (relative L2 <= 5e-3, bf16 output
  = RNE of the FP32 value, max-abs <= 2e-2 rms read per token row).
* Free running.  The GPU's own trajectory of the rows R against the oracle's.  Two correct
  implementations that round differently drift apart; the bound on that drift is derived
  from quantities the test measures on the same layers (see ``free_running_bound``): the
  per-layer discrepancy of the teacher-forced check and the per-layer gain of the block,
  measured in FP64 on the oracle.  The derivation holds while both trajectories route a row
  to the same experts: once the drift tips a near-tie the two compute different functions.
  Each row is therefore compared at its own horizon, the last layer before its first
  routing difference (or the last checked layer).

The chain as configured (x ~ N(0, 1), weights ~ N(0, 0.02), a plain residual add, no
normalisation between blocks) does not stay bounded: a SwiGLU expert grows like |x|^2, so
the residual stream grows faster with every block (rms ~1.2 after 8 blocks, ~3.4 after 21,
~46 after 23) and leaves the FP32 range of the block's arithmetic a few blocks later.  The
block is specified in FP32 (logits, accumulations, the SwiGLU product), so layers are
checked while their values lie well inside that range (|x| and |y| <= 1e15, which keeps
every product inside the block below ~1e33); the test stops at the first layer beyond it
and requires at least MIN_LAYERS checked layers.  Because rows diverge at different rates
(their scales differ by orders of magnitude), max-abs is read per row.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import assert_block_output_rowwise, check_routing, logit_deltas, W_ATOL

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, O.cpu_threads_available()))
LAYERS = 48
MIN_LAYERS = 20       # layers the chain must stay checkable for (inside the FP32 range)
FINITE_LIMIT = 1e15   # largest |x| or |y| of a checked layer
N_TRACK = 64          # rows followed through all layers by the oracle
N_EDGE = 64           # tile-edge rows checked per layer (teacher-forced from the GPU's state)
GAIN_STEP = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from sparse_fp32_softmax_b200.build import build
    build()
    O.build()


def tile_edge_rows(idx, E, exclude, n, seed):
    """Tokens at the first and last row of every 128- and 256-row token tile of every expert
    segment of this routing (the pair tiles' halves and whole tiles), sampled to n."""
    counts, offsets, row_token, _ = O.permute(idx, E, 1)
    edges = set()
    for e in range(E):
        c, o = int(counts[e]), int(offsets[e])
        for tile in (128, 256):
            for s in range(0, c, tile):
                edges.add(int(row_token[o + s]))
                edges.add(int(row_token[o + min(c, s + tile) - 1]))
    edges -= set(exclude)
    edges = sorted(edges)
    rng = np.random.default_rng(seed)
    if len(edges) > n:
        edges = sorted(rng.choice(edges, n, replace=False).tolist())
    return edges


def free_running_bound(inj, gain):
    """Bound on the relative L2 distance after the last layer between two trajectories of
    x_{l+1} = x_l + f_l(x_l) that start equal, follow the same routing, and differ at each
    layer by an injected discrepancy of relative size inj[l] (the GPU's FP32 evaluation and
    its own bf16 rounding against the oracle's, as the teacher-forced check measures it on
    the same layer):
        e_{l+1} <= (1 + gain[l]) e_l + inj[l]      (first order; gain[l] = |df_l| / |dx|)
    so e_L <= sum_l inj[l] * prod_{m > l} (1 + gain[m]).  The discrepancies of the layers
    come from different roundings of different values; they are not aligned, so the
    root-sum-square is the expected size; the bound takes three times it, and never less
    than the largest single term."""
    L = len(inj)
    terms = []
    for l in range(L):
        p = 1.0
        for m in range(l + 1, L):
            p *= 1.0 + gain[m]
        terms.append(inj[l] * p)
    return max(3.0 * math.sqrt(sum(t * t for t in terms)), max(terms))


def test_chain_48_blocks_full_size():
    cfg = inputs.CONFIGS["keras"]
    T, D, E, k = cfg.T, cfg.D, cfg.E, cfg.k
    x0 = inputs.normal_bf16((T, D), 1.0, 1000 * cfg.seed + inputs.TID_X)
    track = inputs.coverage_rows(T, N_TRACK - 2, cfg.seed)[:N_TRACK]
    track_t = torch.tensor(track, dtype=torch.long)
    nt = len(track)
    x_g = x0.cuda()                           # the GPU's free-running state, all rows
    x_o = x0[track_t].clone()                 # the oracle's trajectory of the tracked rows
    dims = B.make_dims(T, D, E, k, cfg.I)
    ws = B.workspace(dims)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    y32 = torch.empty(T, D, dtype=torch.float32, device="cuda")
    idx_free = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.Generator().manual_seed(12345)
    inj, gain, n_checked, n_nondecisive = [], [], 0, 0
    first_diff = {}                           # tracked row -> first layer routed differently
    checked = 0
    XG, XO = [], []                           # tracked rows after each checked layer
    for l in range(LAYERS):
        Wl = inputs.make_layer(cfg, T=T, layer=l, device="cuda", gen_device="cuda", with_x=False)
        Wc = {n: Wl[n].cpu() for n in ("W_r", "W_gate_up", "W_down")}
        # -- teacher-forced pass: tracked rows carry the oracle's trajectory
        x_tf = x_g.clone()
        x_tf[track_t.cuda()] = x_o.cuda()
        row_top = x_tf.float().abs().amax(dim=1).cpu().numpy()
        out = B.moe_forward_ex(x_tf, Wl["W_r"], Wl["W_gate_up"], Wl["W_down"], k, True, ws=ws,
                               residual=x_tf, logits_out=logits, topk_idx_out=idx, topk_w_out=w,
                               out_f32=y32)
        torch.cuda.synchronize()
        assert B.moe_get_device_status(ws) == B.MOE_OK
        idx_h, w_h, logits_h = idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()
        if not np.isfinite(logits_h[track]).all():
            print(f"layer {l}: non-finite router logits on tracked rows, stop")
            break
        fin = np.isfinite(logits_h).all(axis=1)
        o_idx, o_w = O.select(logits_h[fin], k, True)            # selection: every finite token exact
        assert np.array_equal(o_idx, idx_h[fin]), f"layer {l}"
        assert np.abs(o_w - w_h[fin]).max() <= W_ATOL, f"layer {l}"
        # edge rows, among rows whose input lies inside the checked range
        cand = tile_edge_rows(idx_h, E, track, 4 * N_EDGE, 1000 + l)
        edges = [t for t in cand if row_top[t] <= FINITE_LIMIT][:N_EDGE]
        rows = track + edges
        rows_t = torch.tensor(rows, dtype=torch.long)
        x_in = x_tf[rows_t.cuda()].cpu()
        # FP64 gain of the block on every tracked row: f(x + h d) - f(x), |d| = |x|
        d = torch.randn(nt, D, generator=g, dtype=torch.float64)
        xg = x_o.double()
        d *= xg.norm(dim=1, keepdim=True) / d.norm(dim=1, keepdim=True)
        x_pert = (xg + GAIN_STEP * d).to(torch.bfloat16)
        x_all = torch.cat([x_in, x_pert], 0)
        n = len(rows)
        y_all, oi_all, ow_all, ol_all = O.forward_rows(x_all, Wc["W_r"], Wc["W_gate_up"], Wc["W_down"], k,
                                                       list(range(n + nt)), norm=True, residual=x_all,
                                                       threads=THREADS)
        y_o, oi, ol = y_all[:n], oi_all[:n], ol_all[:n]
        top = max(float(row_top[track].max()), float(np.abs(y_o).max()))
        if not np.isfinite(y_o).all() or top > FINITE_LIMIT:
            print(f"layer {l}: checked rows reach |x|,|y| = {top:.3e} > {FINITE_LIMIT:.0e}, stop")
            break
        delta = logit_deltas(x_in, Wc["W_r"], ol)
        assert (np.abs(logits_h[rows] - ol) <= delta + 1e-30).all(), f"layer {l}"
        nd, no = check_routing(idx_h[rows], oi, ol, delta, k)
        n_checked += nd + no
        n_nondecisive += no
        y_ref = y_o.copy()
        diff = [i for i, t in enumerate(rows) if idx_h[t].tolist() != oi[i].tolist()]
        if diff:
            sub = np.asarray(rows, np.int32)[diff]
            y_ref[diff] = O.combine_rows(x_tf.cpu(), idx_h, w_h, sub, Wc["W_gate_up"], Wc["W_down"],
                                         residual=x_tf.cpu(), threads=THREADS)
        yb, yf = out[rows_t.cuda()].cpu(), y32[rows_t.cuda()].cpu()
        rel, worst = assert_block_output_rowwise(yb, yf, y_ref, f"chain layer {l} (teacher-forced)")
        # per row: discrepancy of the tracked rows (GPU bf16 output against the oracle's
        # value, relative to the row's output) and gain of the block; a row whose routing the
        # perturbation changed takes the layer's largest measured gain
        yb_t = yb.double().numpy()[:nt]
        inj.append(np.linalg.norm(yb_t - y_ref[:nt], axis=1) / np.linalg.norm(y_ref[:nt], axis=1))
        keep = np.array([oi_all[n + i].tolist() == oi[i].tolist() for i in range(nt)])
        f0 = y_o[:nt] - xg.numpy()
        f1 = y_all[n:] - x_pert.double().numpy()
        dx = x_pert.double().numpy() - xg.numpy()
        gr = np.linalg.norm(f1 - f0, axis=1) / np.linalg.norm(dx, axis=1)
        gr[~keep] = gr[keep].max() if keep.any() else np.inf
        gain.append(gr)
        e_l = float(np.linalg.norm(yb_t - y_ref[:nt]) / np.linalg.norm(y_ref[:nt]))
        rms_y = float(np.sqrt(np.mean(y_ref[:nt] ** 2)))
        print(f"layer {l}: rms(y) {rms_y:.3e} max|y| {np.abs(y_ref[:nt]).max():.3e} rel L2 {rel:.2e} "
              f"worst row max-abs/row rms {worst:.2e} discrepancy {e_l:.2e} gain max {gain[-1].max():.3f} "
              f"non-decisive {no}/{nd + no}")
        # -- the oracle's trajectory advances by its own bf16-rounded outputs
        x_o = torch.from_numpy(y_o[:nt]).to(torch.bfloat16)
        # -- the GPU's free-running pass
        x_next = torch.empty_like(x_g)
        B.moe_forward_ex(x_g, Wl["W_r"], Wl["W_gate_up"], Wl["W_down"], k, True, ws=ws, out=x_next,
                         residual=x_g, topk_idx_out=idx_free)
        torch.cuda.synchronize()
        x_g = x_next
        # a tracked row whose free-running routing differs from the oracle's trajectory
        fr = idx_free.cpu().numpy()[track]
        for i in range(nt):
            if i not in first_diff and fr[i].tolist() != oi[i].tolist():
                first_diff[i] = l
        checked = l + 1
        XG.append(x_g[track_t.cuda()].cpu().double().numpy())
        XO.append(x_o.double().numpy())
        del Wl, Wc
    assert checked >= MIN_LAYERS, f"only {checked} layers inside the checked range"
    # -- free-running comparison: each row at its horizon h (layers 0..h-1 routed alike)
    horizons, worst = [], 0.0
    for i in range(nt):
        h = first_diff.get(i, checked)
        horizons.append(h)
        if h < 1:
            continue
        rel = np.linalg.norm(XG[h - 1][i] - XO[h - 1][i]) / np.linalg.norm(XO[h - 1][i])
        bound = free_running_bound([inj[m][i] for m in range(h)], [gain[m][i] for m in range(h)])
        worst = max(worst, rel / bound)
        assert rel <= bound, f"row {track[i]}: after {h} layers rel L2 {rel:.3e} > bound {bound:.3e}"
    hz = np.asarray(horizons)
    print(f"chain: {checked} of {LAYERS} layers checked, T={T}; teacher-forced rows checked {n_checked} "
          f"(non-decisive {n_nondecisive}); per-row discrepancy max {max(v.max() for v in inj):.2e} "
          f"mean {np.mean([v.mean() for v in inj]):.2e}; free-running horizons min {hz.min()} "
          f"median {np.median(hz):.0f} max {hz.max()} (rows never routed differently: "
          f"{int((hz == checked).sum())}); largest rel L2 / bound {worst:.3f}")
    assert np.median(hz) >= 2, "free-running routing differs from the oracle's almost at once"
