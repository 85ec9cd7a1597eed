"""The 48-block residual chain of the Keras-default shape at full size (D=2048, E=60, k=4,
I=1408, T=4096): x_{l+1} = x_l + MoE_l(x_l), every block with its own seeded weights.

Rows are independent through the whole chain (a token's output depends only on its own
input), so the oracle follows a subset of rows while the GPU runs the whole batch:

* Teacher forcing, every layer.  The GPU's batch at layer l is its own free-running state
  with the tracked rows R replaced by the oracle's bf16 trajectory.  The GPU output of R,
  and of sampled rows at the edges of this layer's expert tiles (whatever the GPU's own
  state holds there), is checked against the oracle run on exactly the same inputs:
  routing exact on decisive tokens and valid elsewhere, selection from the GPU's own logits
  bit-exact for all 4096 tokens, and the full output criterion (relative L2 <= 5e-3,
  max-abs <= 2e-2 rms before the rounding, bf16 output = RNE of the FP32 value).
* Free running.  The GPU's own 48-layer trajectory of the rows R against the oracle's.
  Two correct implementations that round differently drift apart; the bound on that drift
  is derived from quantities the test measures on the same layers (see
  ``free_running_bound``): the per-layer discrepancy of the teacher-forced check and the
  per-layer gain of the block, measured in FP64 on the oracle.  Rows whose routing differs
  from the oracle's at some layer (a near-tie that the drift tipped over) are counted and
  excluded from the bound: past such a layer the two trajectories compute different
  functions.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_fp32_softmax_b200 import binding as B
from sparse_fp32_softmax_b200 import inputs
from tests.parity_util import assert_block_output, check_routing, logit_deltas, W_ATOL

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, O.cpu_threads_available()))
LAYERS = 48
N_TRACK = 64          # rows followed through all layers by the oracle
N_EDGE = 64           # tile-edge rows checked per layer (teacher-forced from the GPU's state)
N_GAIN = 8            # rows whose block gain is measured per layer
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
    ws = B.workspace(dims, B.make_opts(residual=x_g))
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    y32 = torch.empty(T, D, dtype=torch.float32, device="cuda")
    idx_free = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.Generator().manual_seed(12345)
    inj, gain, n_checked, n_nondecisive = [], [], 0, 0
    flipped = set()
    for l in range(LAYERS):
        Wl = inputs.make_layer(cfg, T=T, layer=l, device="cuda", gen_device="cuda", with_x=False)
        Wc = {n: Wl[n].cpu() for n in ("W_r", "W_gate_up", "W_down")}
        # -- teacher-forced pass: tracked rows carry the oracle's trajectory
        x_tf = x_g.clone()
        x_tf[track_t.cuda()] = x_o.cuda()
        out = B.moe_forward_ex(x_tf, Wl["W_r"], Wl["W_gate_up"], Wl["W_down"], k, True, ws=ws,
                               residual=x_tf, logits_out=logits, topk_idx_out=idx, topk_w_out=w,
                               out_f32=y32)
        torch.cuda.synchronize()
        assert B.moe_get_device_status(ws) == B.MOE_OK
        idx_h, w_h, logits_h = idx.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy()
        o_idx, o_w = O.select(logits_h, k, True)                # selection: every token exact
        assert np.array_equal(o_idx, idx_h), f"layer {l}"
        assert np.abs(o_w - w_h).max() <= W_ATOL, f"layer {l}"
        edges = tile_edge_rows(idx_h, E, track, N_EDGE, 1000 + l)
        rows = track + edges
        rows_t = torch.tensor(rows, dtype=torch.long)
        x_in = x_tf[rows_t.cuda()].cpu()
        # FP64 gain of the block on a few tracked rows: f(x + h d) - f(x), |d| = |x|
        d = torch.randn(N_GAIN, D, generator=g, dtype=torch.float64)
        xg = x_o[:N_GAIN].double()
        d *= xg.norm(dim=1, keepdim=True) / d.norm(dim=1, keepdim=True)
        x_pert = (xg + GAIN_STEP * d).to(torch.bfloat16)
        x_all = torch.cat([x_in, x_pert], 0)
        n = len(rows)
        y_all, oi_all, ow_all, ol_all = O.forward_rows(x_all, Wc["W_r"], Wc["W_gate_up"], Wc["W_down"], k,
                                                       list(range(n + N_GAIN)), norm=True, residual=x_all,
                                                       threads=THREADS)
        y_o, oi, ol = y_all[:n], oi_all[:n], ol_all[:n]
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
        assert_block_output(yb, yf, y_ref, f"chain layer {l} (teacher-forced)")
        # per-layer discrepancy of the tracked rows (GPU bf16 output against the oracle's
        # value), relative to the output, and the gain of the block (same routing only)
        same = [i for i in range(nt) if i not in diff]
        e_l = np.linalg.norm(yb.double().numpy()[same] - y_ref[same]) / np.linalg.norm(y_ref[same])
        inj.append(float(e_l))
        keep = [i for i in range(N_GAIN) if oi_all[n + i].tolist() == oi[i].tolist()]
        f0 = y_o[keep] - xg.numpy()[keep]
        f1 = y_all[n:][keep] - x_pert.double().numpy()[keep]
        dx = x_pert.double().numpy()[keep] - xg.numpy()[keep]
        gain.append(float(np.linalg.norm(f1 - f0) / np.linalg.norm(dx)) if keep else 0.0)
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
            if fr[i].tolist() != oi[i].tolist():
                flipped.add(i)
        del Wl, Wc
    # -- free-running comparison
    xg_f = x_g[track_t.cuda()].cpu().double().numpy()
    xo_f = x_o.double().numpy()
    ok = [i for i in range(nt) if i not in flipped]
    rel = np.linalg.norm(xg_f[ok] - xo_f[ok]) / np.linalg.norm(xo_f[ok])
    per_row = np.linalg.norm(xg_f - xo_f, axis=1) / np.linalg.norm(xo_f, axis=1)
    bound = free_running_bound(inj, gain)
    print(f"chain: {LAYERS} layers, T={T}; teacher-forced rows checked {n_checked} "
          f"(non-decisive {n_nondecisive}); per-layer discrepancy max {max(inj):.2e} "
          f"mean {np.mean(inj):.2e}; gain max {max(gain):.3f} mean {np.mean(gain):.3f}; "
          f"free-running rel L2 {rel:.3e} over {len(ok)} rows (bound {bound:.3e}); "
          f"rows with a routing difference {len(flipped)} (their rel L2 max "
          f"{per_row[sorted(flipped)].max() if flipped else 0:.2e})")
    assert len(ok) >= nt // 2, f"routing differs on {len(flipped)} of {nt} tracked rows"
    assert rel <= bound, (rel, bound)
