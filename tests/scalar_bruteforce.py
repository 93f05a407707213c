"""A pure-Python scalar-loop version of the whole focused step, for micro inputs only.

Used only to pin the oracle: no numpy, no vectorisation, every sum an explicit
loop over Python floats, written from the step's definition independently of
`oracle/`.
"""
import math


def _mat(t):
    return t.double().tolist()


def _rms(x, g, eps):
    ms = sum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [x[i] * r * g[i] for i in range(len(x))]


def _matvec(w, x):
    return [sum(w[o][i] * x[i] for i in range(len(x))) for o in range(len(w))]


def _rope(vec, pos, theta):
    d = len(vec)
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        a = pos * theta ** (-2.0 * i / d)
        c, s = math.cos(a), math.sin(a)
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def _silu(v):
    return v / (1.0 + math.exp(-v))


def scalar_step(shape, model, batch, tau, k_min, k_max, conf_threshold, alpha=1.0):
    L, D, Hq, Hkv, d = shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    G = Hq // Hkv
    eps, theta = shape.rms_eps, shape.rope_theta
    tokens = batch["block_tokens"].tolist()
    mask = batch["mask"].tolist()
    plen = batch["prefix_len"].tolist()
    table = batch["page_table"].tolist()
    pool = batch["kv_pool"].double().tolist()
    cache = batch["ibc"].double().tolist()
    S = len(pool[0][0][0][0])
    N, B = len(tokens), len(tokens[0])
    E = _mat(model["embed"])
    W = {k: [_mat(t) for t in model[k]] for k in ("wqkv", "wo", "wgate", "wup", "wdown")}
    gam = {k: [t.double().tolist() for t in model[k]] for k in ("attn_norm", "mlp_norm")}

    def prefix_kv(b, l, which, g):
        out = []
        for t in range(plen[b]):
            out.append(pool[table[b][t // S]][l][which][g][t % S])
        return out

    def layer(b, l, xs, rows):
        """xs: hidden rows for block positions `rows`; returns new rows + per-(head,row,key) probs."""
        qs, ks, vs = [], [], []
        for r, j in enumerate(rows):
            h = _rms(xs[r], gam["attn_norm"][l], eps)
            qkv = _matvec(W["wqkv"][l], h)
            pos = plen[b] + j
            qs.append([_rope(qkv[hh * d:(hh + 1) * d], pos, theta) for hh in range(Hq)])
            ks.append([_rope(qkv[(Hq + g) * d:(Hq + g + 1) * d], pos, theta) for g in range(Hkv)])
            vs.append([qkv[(Hq + Hkv + g) * d:(Hq + Hkv + g + 1) * d] for g in range(Hkv)])
        for r, j in enumerate(rows):
            for g in range(Hkv):
                cache[b][l][0][g][j] = ks[r][g]
                cache[b][l][1][g][j] = vs[r][g]
        probs = {}
        new = []
        for r, j in enumerate(rows):
            o = []
            for hh in range(Hq):
                g = hh // G
                keys = prefix_kv(b, l, 0, g) + [cache[b][l][0][g][t] for t in range(B)]
                vals = prefix_kv(b, l, 1, g) + [cache[b][l][1][g][t] for t in range(B)]
                sc = [sum(qs[r][hh][i] * kk[i] for i in range(d)) / math.sqrt(d) for kk in keys]
                mx = max(sc)
                ex = [math.exp(s - mx) for s in sc]
                tot = sum(ex)
                p = [e / tot for e in ex]
                probs[(hh, r)] = p
                o.extend(sum(p[t] * vals[t][i] for t in range(len(vals))) for i in range(d))
            x = [xs[r][i] + v for i, v in enumerate(_matvec(W["wo"][l], o))]
            h2 = _rms(x, gam["mlp_norm"][l], eps)
            gt, up = _matvec(W["wgate"][l], h2), _matvec(W["wup"][l], h2)
            a = [_silu(gt[i]) * up[i] for i in range(len(gt))]
            x = [x[i] + v for i, v in enumerate(_matvec(W["wdown"][l], a))]
            new.append(x)
        return new, probs

    xs = [[E[tokens[b][j]][:] for j in range(B)] for b in range(N)]
    imp = [[[0.0] * B for _ in range(N)] for _ in range(2)]
    for l in (0, 1):
        for b in range(N):
            xs[b], probs = layer(b, l, xs[b], list(range(B)))
            for j in range(B):
                imp[l][b][j] = sum(probs[(hh, r)][plen[b] + j] for hh in range(Hq) for r in range(B))
    kept = []
    for b in range(N):
        dl = [imp[1][b][j] - imp[0][b][j] for j in range(B)]
        elig = [j for j in range(B) if mask[b][j]]
        c = sum(1 for j in elig if dl[j] > tau)
        k = min(min(max(math.ceil(alpha * c), k_min), k_max), len(elig))
        # top-k by repeated extraction of the best remaining (largest delta, then smallest j)
        chosen, rest = [], list(elig)
        for _ in range(k):
            best = rest[0]
            for j in rest[1:]:
                if dl[j] > dl[best] or (dl[j] == dl[best] and j < best):
                    best = j
            chosen.append(best)
            rest.remove(best)
        kept.append(sorted(chosen))
    hid = []
    for b in range(N):
        rows = kept[b]
        cur = [xs[b][j] for j in rows]
        for l in range(2, L):
            if rows:
                cur, _ = layer(b, l, cur, rows)
        hid.append(cur)
    gf, lm = model["final_norm"].double().tolist(), _mat(model["lm_head"])
    out = {"importance": imp, "kept": kept, "hidden": hid, "conf": [], "top": [], "decoded": []}
    for b in range(N):
        cf, tp = [], []
        for x in hid[b]:
            z = _matvec(lm, _rms(x, gf, eps))
            best = 0
            for i in range(1, len(z)):
                if z[i] > z[best]:
                    best = i
            cf.append(1.0 / sum(math.exp(v - z[best]) for v in z))
            tp.append(best)
        dec = {}
        cand = [t for t, j in enumerate(kept[b]) if mask[b][j]]
        for t in cand:
            if cf[t] > conf_threshold:
                dec[kept[b][t]] = tp[t]
        if not dec and cand:
            best = cand[0]
            for t in cand[1:]:
                if cf[t] > cf[best]:
                    best = t
            dec[kept[b][best]] = tp[best]
        out["conf"].append(cf)
        out["top"].append(tp)
        out["decoded"].append(dec)
    out["cache"] = cache
    return out
