"""An independently written dense block forward, used only to pin the oracle.

It shares no code with `oracle/`: torch float64 ops, RoPE as a complex-number
rotation, attention through torch's scaled_dot_product_attention with the KV
heads repeated for the grouped query heads.  With every position kept (forced
keep fraction 1) the focused step must reduce to exactly this computation.
"""
import torch
import torch.nn.functional as F


def _rms(x, g, eps):
    return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + eps) * g


def _rope_complex(x, pos, theta):
    # pair (i, i + d/2) as the complex number x_i + 1j * x_{i+d/2}, turned by e^{1j * pos * theta^(-2i/d)}
    d = x.shape[-1]
    half = d // 2
    freq = torch.pow(torch.tensor(theta, dtype=torch.float64), -torch.arange(0, d, 2, dtype=torch.float64) / d)
    turn = torch.polar(torch.ones(len(pos), half, dtype=torch.float64), pos[:, None].double() * freq[None, :])
    z = torch.complex(x[..., :half], x[..., half:]) * turn
    return torch.cat([z.real, z.imag], dim=-1)


def dense_block_forward(shape, model, batch):
    """Run all L layers on every block row of every request.

    Returns dict with per-request final hidden rows [N, B, D], logits [N, B, V],
    the block K/V of every layer [N, L, 2, Hkv, B, d] and the layer-0/1 full
    attention probabilities' block-column sums [2, N, B].
    """
    f64 = lambda t: t.detach().to("cpu", torch.float64)
    tokens = batch["block_tokens"].long().cpu()
    plen = batch["prefix_len"].long().cpu()
    table = batch["page_table"].long().cpu()
    pool = batch["kv_pool"]
    N, B = tokens.shape
    L, D, Hq, Hkv, d = shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    G = Hq // Hkv
    S = pool.shape[4]
    hidden = torch.empty(N, B, D, dtype=torch.float64)
    kv = torch.empty(N, L, 2, Hkv, B, d, dtype=torch.float64)
    colsum = torch.zeros(2, N, B, dtype=torch.float64)
    logits = []
    for b in range(N):
        P = int(plen[b])
        pos = torch.arange(P, P + B)
        x = f64(model["embed"])[tokens[b]]
        for l in range(L):
            h = _rms(x, f64(model["attn_norm"][l]), shape.rms_eps)
            qkv = h @ f64(model["wqkv"][l]).T
            q = qkv[:, : Hq * d].view(B, Hq, d).permute(1, 0, 2)
            k = qkv[:, Hq * d:(Hq + Hkv) * d].view(B, Hkv, d).permute(1, 0, 2)
            v = qkv[:, (Hq + Hkv) * d:].view(B, Hkv, d).permute(1, 0, 2)
            q = _rope_complex(q, pos, shape.rope_theta)
            k = _rope_complex(k, pos, shape.rope_theta)
            kv[b, l, 0], kv[b, l, 1] = k, v
            if P > 0:
                slots = torch.arange(P)
                pages = table[b, slots // S]
                pk = f64(pool[pages, l, 0][:, :, :].permute(1, 0, 2, 3))  # [Hkv, P, S, d]
                pv = f64(pool[pages, l, 1][:, :, :].permute(1, 0, 2, 3))
                pk = pk[:, torch.arange(P), slots % S]
                pv = pv[:, torch.arange(P), slots % S]
                keys, vals = torch.cat([pk, k], 1), torch.cat([pv, v], 1)
            else:
                keys, vals = k, v
            keys = keys.repeat_interleave(G, dim=0)
            vals = vals.repeat_interleave(G, dim=0)
            o = F.scaled_dot_product_attention(q[None], keys[None], vals[None])[0]
            if l < 2:
                probs = torch.softmax(q @ keys.transpose(1, 2) / d ** 0.5, dim=-1)
                colsum[l, b] = probs[:, :, P:].sum(dim=(0, 1))
            x = x + o.permute(1, 0, 2).reshape(B, Hq * d) @ f64(model["wo"][l]).T
            h2 = _rms(x, f64(model["mlp_norm"][l]), shape.rms_eps)
            a = F.silu(h2 @ f64(model["wgate"][l]).T) * (h2 @ f64(model["wup"][l]).T)
            x = x + a @ f64(model["wdown"][l]).T
        hidden[b] = x
        hf = _rms(x, f64(model["final_norm"]), shape.rms_eps)
        logits.append(hf @ f64(model["lm_head"]).T)
    return {"hidden": hidden, "logits": torch.stack(logits), "kv": kv, "colsum": colsum}
