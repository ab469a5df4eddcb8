"""Teacher-forced parity check of cq_moe_ffn against the CPU oracle.

Each oracle stage takes the GPU's previous-stage output, so that a quantized
code is compared against the oracle's decision for exactly the same input:
  x codes/scales         bit-exact
  routing tables         bit-exact (ids, counts, offsets, perm); weights ~1e-6
  h = fp16(silu(g) u)    within the tolerance propagated from g, u + 1 fp16 ulp
  h codes/scales         bit-exact (oracle rotate+quantize of the GPU's h)
  y per row              |y - y_ref| <= 1e-4 * s * sum|C q| + 1e-6
  out                    fp32 combine of the GPU's y and weights
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


_CACHE: dict = {}


def moe_inputs_cached(shape, seed=0):
    """Inputs of one workload, generated once per test session."""
    key = (repr(shape), seed)
    if key not in _CACHE:
        if len(_CACHE) >= 3:
            _CACHE.pop(next(iter(_CACHE)))
        _CACHE[key] = synth.moe_inputs(shape, seed=seed)
    return _CACHE[key]


def cfg_of(s: synth.MoEShape):
    import lut_clustered_weight_b200 as cq
    return cq.MoEConfig(H=s.H, I=s.I, E=s.E, top_k=s.top_k, n_shared=s.n_shared,
                        I_shared=s.I_shared, act_bits=s.act_bits, had_block_h=s.had_block_h,
                        had_block_i=s.had_block_i, had_block_i_shared=s.had_block_i_shared,
                        renormalize=s.renormalize)


def upload_weights(inp: synth.MoEInputs, dev):
    w = {}
    for n in ("gate_idx", "up_idx", "down_idx", "gate_cb", "up_cb", "down_cb", "sh_gate_idx",
              "sh_up_idx", "sh_down_idx", "sh_gate_cb", "sh_up_cb", "sh_down_cb"):
        a = getattr(inp, n)
        if a is not None:
            w[n] = torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    for n in ("x_scale", "x_perm"):   # online smoothing scale / channel order of x
        if inp.extra.get(n) is not None:
            w[n] = torch.from_numpy(np.ascontiguousarray(inp.extra[n])).to(dev)
    return w


def run_moe(inp: synth.MoEInputs, dev="cuda", debug=True):
    import lut_clustered_weight_b200 as cq
    s = inp.shape
    cfg = cfg_of(s)
    T, H = s.T, s.H
    Rr = T * s.top_k if s.E else 0
    R = Rr + s.n_shared * T
    Imax = max(s.I if s.E else 0, s.I_shared if s.n_shared else 0)
    cb = (lambda K: K // 2 if s.act_bits == 4 else K)
    cdt = torch.uint8 if s.act_bits == 4 else torch.int8
    x = torch.from_numpy(inp.x).to(dev)
    lg = torch.from_numpy(inp.logits).to(dev) if s.E else None
    w = upload_weights(inp, dev)
    dbg = None
    if debug:
        dbg = dict(
            topk_ids=torch.full((max(Rr, 1),), -1, dtype=torch.int32, device=dev),
            topk_w=torch.zeros((max(Rr, 1),), dtype=torch.float32, device=dev),
            counts=torch.full((max(s.E, 1),), -1, dtype=torch.int32, device=dev),
            offsets=torch.full((s.E + 1,), -1, dtype=torch.int32, device=dev),
            perm=torch.full((max(Rr, 1),), -1, dtype=torch.int32, device=dev),
            x_codes=torch.zeros((T, cb(H)), dtype=cdt, device=dev),
            x_scales=torch.zeros((T,), dtype=torch.float32, device=dev),
            h=torch.zeros((R, Imax), dtype=torch.float16, device=dev),
            h_codes=torch.zeros((R, cb(Imax)), dtype=cdt, device=dev),
            h_scales=torch.zeros((R,), dtype=torch.float32, device=dev),
            y_rows=torch.zeros((R, H), dtype=torch.float32, device=dev),
        )
        if not s.E:
            for k in ("topk_ids", "topk_w", "counts", "offsets", "perm"):
                dbg[k] = None
    out = cq.cq_moe_ffn(cfg, x, lg, w, debug=dbg)
    torch.cuda.synchronize()
    res = {"out": out.cpu().numpy()}
    if dbg:
        for k, v in dbg.items():
            if v is not None:
                res[k] = v.cpu().numpy()
    return res


def _rows_of(s, g):
    """(row -> (token, expert or -1-shared)) for the internal row order."""
    rows = []
    if s.E:
        perm = g["perm"]
        ids = g["topk_ids"]
        for p in range(s.T * s.top_k):
            sl = int(perm[p])
            rows.append((sl // s.top_k, int(ids[sl])))
    for sh in range(s.n_shared):
        for t in range(s.T):
            rows.append((t, -1 - sh))
    return rows


def check_moe(inp: synth.MoEInputs, g: dict, *, sample_rows=None, sample_tokens=None,
              e2e=False, rng_seed=0):
    """Assert teacher-forced parity; returns a dict of error statistics."""
    s = inp.shape
    bits = s.act_bits
    stats = {}
    # -- x codes and scales (bit-exact)
    xq_ref, sx_ref = oracle.rotate_quantize(inp.x, s.had_block_h, bits,
                                            scale=inp.extra.get("x_scale"),
                                            perm=inp.extra.get("x_perm"))
    xq = oracle.unpack_codes(g["x_codes"], s.H, bits)
    assert np.array_equal(xq, xq_ref), "x codes differ"
    assert np.array_equal(g["x_scales"].view(np.uint32), sx_ref.view(np.uint32)), "x scales differ"
    # -- routing (bit-exact tables)
    if s.E:
        rt = oracle.route(inp.logits, s.top_k, bool(s.renormalize))
        assert np.array_equal(g["topk_ids"].reshape(s.T, s.top_k), rt["ids"]), "top-k ids differ"
        assert np.array_equal(g["counts"], rt["counts"]), "counts differ"
        assert np.array_equal(g["offsets"], rt["offsets"]), "offsets differ"
        assert np.array_equal(g["perm"], rt["perm"]), "perm differs"
        werr = np.abs(g["topk_w"].reshape(s.T, s.top_k) - rt["w"])
        assert np.all(werr <= 2e-6 * np.abs(rt["w"]) + 1e-7), f"weights differ {werr.max()}"
        stats["w_max_err"] = float(werr.max())
    rows = _rows_of(s, g)
    R = len(rows)
    rng = np.random.default_rng(rng_seed)
    if sample_rows is None:
        sel = np.arange(R)
    else:
        sel = np.unique(np.concatenate([[0, R - 1], rng.choice(R, min(sample_rows, R),
                                                                replace=False)]))

    def W(expert, which):
        if expert >= 0:
            return getattr(inp, f"{which}_idx")[expert], getattr(inp, f"{which}_cb")[expert]
        sh = -1 - expert
        return getattr(inp, f"sh_{which}_idx")[sh], getattr(inp, f"sh_{which}_cb")[sh]

    h_worst = y_worst = 0.0
    for p in sel:
        t, ex = rows[p]
        I_r = s.I if ex >= 0 else s.I_shared
        b_i = s.had_block_i if ex >= 0 else s.had_block_i_shared
        xr = xq[t:t + 1]
        sxr = g["x_scales"][t:t + 1]
        gr, gm, _ = oracle.lut_gemm(xr, sxr, *W(ex, "gate"))
        ur, um, _ = oracle.lut_gemm(xr, sxr, *W(ex, "up"))
        tg, tu = oracle.lut_tolerance(gm), oracle.lut_tolerance(um)
        h_ref = oracle.swiglu(gr, ur).astype(np.float64)[0]
        hg = g["h"][p, :I_r].astype(np.float64)
        sig = 1.0 / (1.0 + np.exp(-gr[0]))
        bound = (1.1 * np.abs(ur[0]) * tg[0] + np.abs(gr[0] * sig) * tu[0] + tg[0] * tu[0]
                 + np.spacing(np.abs(h_ref).astype(np.float16)).astype(np.float64) + 1e-6)
        herr = np.abs(hg - h_ref)
        assert np.all(herr <= bound), f"h row {p}: max excess {(herr - bound).max()}"
        h_worst = max(h_worst, float((herr / bound).max()))
        # h codes / scales from the GPU's h (bit-exact)
        hq_ref, sh_ref = oracle.rotate_quantize(g["h"][p:p + 1, :I_r], b_i, bits)
        hq = oracle.unpack_codes(g["h_codes"][p:p + 1, :(I_r // 2 if bits == 4 else I_r)],
                                 I_r, bits)
        assert np.array_equal(hq, hq_ref), f"h codes row {p} differ"
        assert g["h_scales"][p].view(np.uint32) == sh_ref.view(np.uint32)[0], f"h scale row {p}"
        # down-projection row
        yr, ym, _ = oracle.lut_gemm(hq, g["h_scales"][p:p + 1], *W(ex, "down"))
        yerr = np.abs(g["y_rows"][p].astype(np.float64) - yr[0])
        ytol = oracle.lut_tolerance(ym[0])
        assert np.all(yerr <= ytol), f"y row {p}: max excess {(yerr - ytol).max()}"
        y_worst = max(y_worst, float((yerr / ytol).max()))
    stats["h_err_over_bound"] = h_worst
    stats["y_err_over_bound"] = y_worst
    # -- combine, from the GPU's y rows and weights
    toks = np.arange(s.T) if sample_tokens is None else np.unique(
        np.concatenate([[0, s.T - 1], rng.choice(s.T, min(sample_tokens, s.T), replace=False)]))
    yrows = g["y_rows"].astype(np.float64)
    Rr = s.T * s.top_k if s.E else 0
    if s.E:
        inv = np.empty(Rr, dtype=np.int64)
        inv[g["perm"]] = np.arange(Rr)
        wg = g["topk_w"].reshape(s.T, s.top_k).astype(np.float64)
    out_err = 0.0
    for t in toks:
        terms = []
        for j in range(s.top_k if s.E else 0):
            terms.append(wg[t, j] * yrows[inv[t * s.top_k + j]])
        for sh in range(s.n_shared):
            terms.append(yrows[Rr + sh * s.T + t])
        terms = np.array(terms)
        ref = terms.sum(0)
        tol = 4e-7 * np.abs(terms).sum(0) * max(len(terms), 1) + 1e-6
        err = np.abs(g["out"][t] - ref)
        assert np.all(err <= tol), f"out token {t}: max excess {(err - tol).max()}"
        out_err = max(out_err, float((err / tol).max()))
    stats["out_err_over_bound"] = out_err
    if e2e:
        ref = oracle.moe_ffn(inp)["out"]
        rel = float(np.linalg.norm(g["out"] - ref) / max(np.linalg.norm(ref), 1e-30))
        stats["e2e_rel_l2"] = rel
    return stats
