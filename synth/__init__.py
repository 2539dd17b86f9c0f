"""Seeded synthetic inputs for the Fathom key scan.

This module is the one piece of code that both the oracle side (tests, CPU
baseline) and the CUDA side (tests, bench) use.  It draws inputs and converts
data types; it holds none of the method's arithmetic (no quantizer, no
planes, no depths, no scores).

Recipe (the pages give only shapes; distributions are stated as readings):
  * per (KV head, channel) scale sigma_c = exp(U(ln 0.1, ln 3)); 4 outlier
    channels per KV head, drawn without replacement, get sigma_c *= 8;
  * keys x ~ N(0, sigma_c^2) in fp32, shape [Hkv][n][d];
  * queries q ~ N(0, 1) per channel, shape [Hq][d];
  * values V ~ N(0, 1), stored as bf16, shape [Hkv][n][d];
  * sigma2 (the "offline statistic") = fp64 mean of x^2 over a KV head's
    keys, rounded to fp32;
  * seed = 1000 * config + layer.
"""
import numpy as np

LOG_LO, LOG_HI = np.log(0.1), np.log(3.0)
N_OUTLIERS = 4
OUTLIER_MULT = 8.0


def rng_for(config, layer=0, stream=0):
    """numpy Generator for (config, layer); `stream` separates independent draws."""
    return np.random.Generator(np.random.PCG64([1000 * int(config) + int(layer), int(stream)]))


def channel_sigma(rng, n_kv_heads, d, n_outliers=N_OUTLIERS, mult=OUTLIER_MULT):
    sig = np.exp(rng.uniform(LOG_LO, LOG_HI, size=(n_kv_heads, d)))
    for g in range(n_kv_heads):
        if n_outliers:
            ch = rng.choice(d, size=min(n_outliers, d), replace=False)
            sig[g, ch] *= mult
    return sig


def keys(rng, sigma, n, out=None, chunk=1 << 16):
    """fp32 keys [Hkv][n][d], x ~ N(0, sigma_c^2), generated in key chunks."""
    Hkv, d = sigma.shape
    if out is None:
        out = np.empty((Hkv, n, d), np.float32)
    sig32 = sigma.astype(np.float32)
    for g in range(Hkv):
        for i0 in range(0, n, chunk):
            i1 = min(n, i0 + chunk)
            z = rng.standard_normal((i1 - i0, d), dtype=np.float32)
            np.multiply(z, sig32[g][None, :], out=out[g, i0:i1])
    return out


def queries(rng, n_q_heads, d):
    return rng.standard_normal((n_q_heads, d)).astype(np.float32)


def f32_to_bf16_bits(x):
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def values_bf16(rng, n_kv_heads, n, d, chunk=1 << 16):
    out = np.empty((n_kv_heads, n, d), np.uint16)
    for g in range(n_kv_heads):
        for i0 in range(0, n, chunk):
            i1 = min(n, i0 + chunk)
            out[g, i0:i1] = f32_to_bf16_bits(rng.standard_normal((i1 - i0, d), dtype=np.float32))
    return out


def sigma2_of_keys(K):
    """fp64 mean of x^2 over each KV head's keys, rounded to fp32: [Hkv][d]."""
    Hkv, n, d = K.shape
    s = np.zeros((Hkv, d), np.float64)
    for g in range(Hkv):
        for i0 in range(0, n, 1 << 16):
            blk = K[g, i0:i0 + (1 << 16)].astype(np.float64)
            s[g] += np.einsum("ij,ij->j", blk, blk)
    return (s / max(n, 1)).astype(np.float32)


def needle_positions(rng, n, count=16):
    return np.sort(rng.choice(n, size=count, replace=False))


def needle_rows(rng, rows, q_head, cosine=0.9):
    """New key rows for needles: |k_orig| * (cosine * q_hat + sqrt(1 - cosine^2) * u_perp),
    u_perp a random unit vector orthogonal to q.  rows: [count][d] originals."""
    qv = np.asarray(q_head, np.float64)
    q_hat = qv / np.linalg.norm(qv)
    out = np.empty(rows.shape, np.float32)
    for e in range(rows.shape[0]):
        u = rng.standard_normal(qv.size)
        u -= u.dot(q_hat) * q_hat
        u /= np.linalg.norm(u)
        out[e] = np.linalg.norm(rows[e].astype(np.float64)) * (cosine * q_hat + np.sqrt(1 - cosine * cosine) * u)
    return out


def plant_needles(rng, K, q_head, kv_head=0, count=16, cosine=0.9):
    """Overwrite `count` seeded key positions of `kv_head` with needles; returns the positions."""
    pos = needle_positions(rng, K.shape[1], count)
    K[kv_head, pos] = needle_rows(rng, K[kv_head, pos], q_head, cosine)
    return pos


# Workload shapes (one KV layer).  Budgets, k and residency as the workloads state.
CONFIGS = {
    1: dict(name="single-head n=4096 d=128 B=64 k=64 hbm", n_kv_heads=1, n_q_heads=1, d=128, n=4096,
            budgets=(64,), k=64, q_dtype="f32", resident="hbm"),
    2: dict(name="qwen3-8b layer n=131072 B={46,68,92,136} k=2048 hbm", n_kv_heads=8, n_q_heads=32, d=128,
            n=131072, budgets=(46, 68, 92, 136), k=2048, q_dtype="bf16", resident="hbm"),
    3: dict(name="qwen3-8b layer n=1048576 B=92 k=2048 host-resident, 16 needles", n_kv_heads=8, n_q_heads=32,
            d=128, n=1048576, budgets=(92,), k=2048, q_dtype="bf16", resident="host", needles=16),
    4: dict(name="16 sessions n~U[64k,512k] B=68 k=1024 host-resident", n_kv_heads=8, n_q_heads=32, d=128,
            sessions=16, n_lo=65536, n_hi=524288, budgets=(68,), k=1024, q_dtype="bf16", resident="host"),
    5: dict(name="36-layer qwen3-8b decode n=1048576 B~U[46,136] k=2048 host-resident", n_kv_heads=8,
            n_q_heads=32, d=128, n=1048576, layers=36, b_lo=46, b_hi=136, k=2048, q_dtype="bf16",
            resident="host"),
}


def layer_inputs(config, layer=0, n=None, n_kv_heads=None, n_q_heads=None, d=None, with_values=False,
                 needles=None):
    """All inputs of one layer of a workload: dict of numpy arrays.

    Keys are returned in fp32 (the packer's input) and as bf16 rows (the
    attention's input).  q is fp32 for f32 workloads and bf16-rounded
    (returned widened, plus its bf16 bits) otherwise.
    """
    cfg = CONFIGS[config]
    n = cfg.get("n", 4096) if n is None else n
    Hkv = cfg["n_kv_heads"] if n_kv_heads is None else n_kv_heads
    Hq = cfg["n_q_heads"] if n_q_heads is None else n_q_heads
    d = cfg["d"] if d is None else d
    rs = rng_for(config, layer, 0)
    sigma = channel_sigma(rs, Hkv, d)
    K = keys(rng_for(config, layer, 1), sigma, n)
    q = queries(rng_for(config, layer, 2), Hq, d)
    out = {}
    if cfg["q_dtype"] == "bf16":
        qb = f32_to_bf16_bits(q)
        out["q_bf16"] = qb
        q = bf16_bits_to_f32(qb)
    out["q"] = q
    nd = cfg.get("needles", 0) if needles is None else needles
    if nd:
        out["needles"] = plant_needles(rng_for(config, layer, 3), K, q[0], kv_head=0, count=nd)
    out["K"] = K
    out["sigma2"] = sigma2_of_keys(K)
    if with_values:
        out["K_rows"] = f32_to_bf16_bits(K)
        out["V_rows"] = values_bf16(rng_for(config, layer, 4), Hkv, n, d)
    return out


def layer_inputs_cuda(config, layer=0, n=None, n_kv_heads=None, n_q_heads=None, d=None, device="cuda",
                      with_values=True, needles=None, part=0):
    """One layer of a workload generated on the GPU (torch's Philox generator,
    seeded like the numpy path): same recipe, different draws.  Returns torch
    tensors on `device`: K f32, K_rows/V_rows bf16 [Hkv][n][d], q (f32 or bf16)
    [Hq][d], sigma2 f32 [Hkv][d]; plus numpy copies of q and sigma2 and the
    needle positions.  part > 0 draws the keys and values of another key range
    of the same layer (same channel scales and queries; sigma2 is then that
    range's own statistic)."""
    import torch
    cfg = CONFIGS[config]
    n = cfg.get("n", 4096) if n is None else n
    Hkv = cfg["n_kv_heads"] if n_kv_heads is None else n_kv_heads
    Hq = cfg["n_q_heads"] if n_q_heads is None else n_q_heads
    d = cfg["d"] if d is None else d
    sigma = channel_sigma(rng_for(config, layer, 0), Hkv, d)
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 * int(config) + int(layer) + 1000003 * int(part))
    K = torch.empty((Hkv, n, d), dtype=torch.float32, device=device)
    sig_t = torch.from_numpy(sigma.astype(np.float32)).to(device)
    for g in range(Hkv):
        K[g].normal_(generator=gen)
        K[g].mul_(sig_t[g][None, :])
    q = queries(rng_for(config, layer, 2), Hq, d)
    out = {}
    if cfg["q_dtype"] == "bf16":
        qb = f32_to_bf16_bits(q)
        q = bf16_bits_to_f32(qb)
        out["q_dev"] = torch.from_numpy(qb.view(np.int16)).to(device).view(torch.bfloat16)
    else:
        out["q_dev"] = torch.from_numpy(q).to(device)
    out["q"] = q
    nd = cfg.get("needles", 0) if needles is None else needles
    if nd:
        rng = rng_for(config, layer, 3)
        pos = needle_positions(rng, n, nd)
        rows = K[0, torch.from_numpy(pos).to(device)].cpu().numpy()
        K[0, torch.from_numpy(pos).to(device)] = torch.from_numpy(needle_rows(rng, rows, q[0])).to(device)
        out["needles"] = pos
    s2 = torch.empty((Hkv, d), dtype=torch.float64, device=device)
    for g in range(Hkv):
        s2[g] = K[g].double().square().mean(dim=0)
    out["sigma2_dev"] = s2.float()
    out["sigma2"] = out["sigma2_dev"].cpu().numpy()
    out["K"] = K
    if with_values:
        out["K_rows"] = K.to(torch.bfloat16)
        V = torch.empty((Hkv, n, d), dtype=torch.bfloat16, device=device)
        for g in range(Hkv):
            V[g].normal_(generator=gen)
        out["V_rows"] = V
    return out
