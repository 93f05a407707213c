"""An independently written dense block forward, used only to pin the oracle.

It shares no code with `oracle/`: torch ops, RoPE as a complex-number rotation, attention through
torch's scaled_dot_product_attention (or written out, when the probabilities are rounded) with the KV
heads repeated for the grouped query heads.  With every position kept (forced keep fraction 1) the
focused step must reduce to exactly this computation.

Two knobs make it a second, independent bf16 evaluation of the same model:
  * storage="bf16" rounds to bfloat16 where a bf16 kernel stores activations: the normalised rows (before
    QKV, before the MLP, before the LM head), q and k after RoPE, v, the attention output and the SwiGLU
    product; the residual stream is never rounded;
  * accum="f32" runs every product, softmax and norm in float32 (as tensor-core kernels accumulate), and
    round_probs=True rounds the unnormalised softmax weights to bf16 before they multiply V (as a
    tensor-core P.V product takes them), while the denominator keeps the float32 values.
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
    z = torch.complex(x[..., :half].double(), x[..., half:].double()) * turn
    return torch.cat([z.real, z.imag], dim=-1).to(x.dtype)


def _to_bf16_and_back(t):
    return t.to(torch.bfloat16).to(t.dtype)


def _attend(q, keys, vals, round_probs, store):
    """softmax(q k^T / sqrt(d)) v per head; with round_probs the weights e = exp(s - max) meet V in bf16."""
    d = q.shape[-1]
    if not round_probs:
        return F.scaled_dot_product_attention(q[None], keys[None], vals[None])[0]
    s = q @ keys.transpose(1, 2) / d ** 0.5
    e = torch.exp(s - s.amax(-1, keepdim=True))
    return (store(e) @ vals) / e.sum(-1, keepdim=True)


def dense_block_forward(shape, model, batch, storage="f64", accum="f64", round_probs=False, requests=None):
    """Run all L layers on every block row of every request (or of `requests`).

    Returns dict with per-request final hidden rows [N, B, D], logits [N, B, V],
    the block K/V of every layer [N, L, 2, Hkv, B, d] and the layer-0/1 full
    attention probabilities' block-column sums [2, N, B] (all float64 tensors).
    """
    dt = torch.float64 if accum == "f64" else torch.float32
    cv = lambda t: t.detach().to("cpu", dt)
    store = _to_bf16_and_back if storage == "bf16" else (lambda t: t)
    reqs = list(range(batch["block_tokens"].shape[0])) if requests is None else list(requests)
    tokens = batch["block_tokens"].long().cpu()[reqs]
    plen = batch["prefix_len"].long().cpu()[reqs]
    table = batch["page_table"].long().cpu()[reqs]
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
        x = cv(model["embed"])[tokens[b]]
        for l in range(L):
            h = store(_rms(x, cv(model["attn_norm"][l]), shape.rms_eps))
            qkv = h @ cv(model["wqkv"][l]).T
            q = qkv[:, : Hq * d].view(B, Hq, d).permute(1, 0, 2)
            k = qkv[:, Hq * d:(Hq + Hkv) * d].view(B, Hkv, d).permute(1, 0, 2)
            v = store(qkv[:, (Hq + Hkv) * d:].view(B, Hkv, d).permute(1, 0, 2))
            q = store(_rope_complex(q, pos, shape.rope_theta))
            k = store(_rope_complex(k, pos, shape.rope_theta))
            kv[b, l, 0], kv[b, l, 1] = k.double(), v.double()
            if P > 0:
                slots = torch.arange(P)
                pages = table[b, slots // S]
                pk = cv(pool[pages.to(pool.device), l, 0]).permute(1, 0, 2, 3)  # [Hkv, P, S, d]
                pv = cv(pool[pages.to(pool.device), l, 1]).permute(1, 0, 2, 3)
                pk = pk[:, torch.arange(P), slots % S]
                pv = pv[:, torch.arange(P), slots % S]
                keys, vals = torch.cat([pk, k], 1), torch.cat([pv, v], 1)
            else:
                keys, vals = k, v
            keys = keys.repeat_interleave(G, dim=0)
            vals = vals.repeat_interleave(G, dim=0)
            o = store(_attend(q, keys, vals, round_probs, store))
            if l < 2:
                probs = torch.softmax(q @ keys.transpose(1, 2) / d ** 0.5, dim=-1)
                colsum[l, b] = probs[:, :, P:].sum(dim=(0, 1)).double()
            x = x + o.permute(1, 0, 2).reshape(B, Hq * d) @ cv(model["wo"][l]).T
            h2 = store(_rms(x, cv(model["mlp_norm"][l]), shape.rms_eps))
            a = store(F.silu(h2 @ cv(model["wgate"][l]).T) * (h2 @ cv(model["wup"][l]).T))
            x = x + a @ cv(model["wdown"][l]).T
        hidden[b] = x.double()
        hf = store(_rms(x, cv(model["final_norm"]), shape.rms_eps))
        logits.append((hf @ cv(model["lm_head"]).T).double())
    return {"hidden": hidden, "logits": torch.stack(logits), "kv": kv, "colsum": colsum}
