"""Error budget of the tensor-core projection's second product: the gated low-rank operand
g_j dt_low^j (fp32 accumulations of bf16 x and W_x) enters the MMA as bf16, and the projection
carries it as two bf16 parts, hi = bf16(v) and lo = bf16(v - hi) (about 16 significant bits),
at the cost of doubling that product's MMAs. This CPU test measures, with the fp64 oracle on the
Mamba-1.4B-like shape (its weight statistics, 256 tokens of two sequences, sampled channels), what
each choice does to Delta and to the layer output:
* hi alone (8 significant bits) moves the state-space part of y by a sizeable fraction of the
  layer's bf16 tolerance of 2e-2 (measured ~8e-3: a margin under 10x), so the lo part is kept;
* hi + lo leaves an error two orders of magnitude below the tolerance."""
import numpy as np

from oracle import swimba_oracle as O
from parameter_space_moe_swimba_b200 import synth
from parameter_space_moe_swimba_b200.configs import CONFIGS


def test_gated_low_rank_operand_keeps_its_low_bf16_part():
    cfg = CONFIGS["mamba1p4b_like"].with_(batch=2, seqlen=256)
    w = synth.draw_weights(cfg)
    x, z = synth.draw_activations(cfg)
    x64, z64 = synth.widen(x, "bf16"), synth.widen(z, "bf16")
    W_x, W_dt = synth.widen(w.W_x, "bf16"), synth.widen(w.W_dt, "bf16")
    b_dt, A, Dsk = w.b_dt.astype(np.float64), w.A.astype(np.float64), w.D_skip.astype(np.float64)
    B, L, D = x64.shape
    R, N, k = cfg.dt_rank, cfg.d_state, cfg.top_k
    idx, g, _ = O.route(x64.reshape(-1, D), w.W_r.astype(np.float64), k)
    pr = O.expert_projections(x64.reshape(-1, D), idx, g, W_x, W_dt, b_dt, R, N)
    dt_low = pr["xdbl"][:, :, :R]  # [T, k, R]
    v = g[:, :, None] * dt_low
    hi = synth.widen(synth.round_to(v, "bf16"), "bf16")  # round to nearest even
    lo = synth.widen(synth.round_to(v - hi, "bf16"), "bf16")
    exact = pr["dt_mix"]
    ch = np.arange(0, D, 37)
    shp = lambda a: a.reshape(B, L, *a.shape[1:])
    args = (shp(pr["B_mix"]), shp(pr["C_mix"]), shp(idx), shp(g), A, Dsk)
    y0, *_ = O.selective_scan(x64, z64, shp(exact), *args, channels=ch)
    ssm0 = y0 - Dsk[ch] * x64[:, :, ch]
    d_exact = O.softplus(exact)

    def errors(op):
        dt_mix = np.zeros((B * L, D))
        for j in range(k):
            for e in range(cfg.n_experts):
                rows = np.nonzero(idx[:, j] == e)[0]
                dt_mix[rows] += op[rows, j] @ W_dt[e] + g[rows, j, None] * b_dt[e]
        d = O.softplus(dt_mix)
        y1, *_ = O.selective_scan(x64, z64, shp(dt_mix), *args, channels=ch)
        ssm1 = y1 - Dsk[ch] * x64[:, :, ch]
        return {
            "delta": np.max(np.abs(d - d_exact) / (np.sqrt(np.mean(d_exact ** 2)) + np.abs(d_exact))),
            "y": np.max(np.abs(y1 - y0) / (1 + np.abs(y0))),
            "y_ssm": np.max(np.abs(ssm1 - ssm0) / (np.sqrt(np.mean(ssm0 ** 2)) + np.abs(ssm0))),
        }

    e_hi, e_hilo = errors(hi), errors(hi + lo)
    print({"hi": e_hi, "hi+lo": e_hilo})
    assert e_hi["y_ssm"] > 2e-3  # hi alone: less than a tenfold margin under 2e-2
    assert e_hi["y_ssm"] < 2e-2
    assert max(e_hilo.values()) < 2e-4  # hi + lo: a hundredfold margin
