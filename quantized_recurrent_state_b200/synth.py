"""Seeded synthetic workloads (inputs only; no STEPQuant arithmetic here).

Shared by the tests, the benchmark and the CPU reference checks: it draws
random numbers and shapes them; it never quantizes, updates or reads out a
state.  Random numbers come from a counter-based SplitMix64 stream
(Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014: state += 0x9E3779B97F4A7C15, then the xor-shift-multiply
finalizer), turned into uniforms with the top 53 bits and into normals with
the Box-Muller transform.  The numpy path is exact and host-side; the torch
path runs the same integer stream on a CUDA device (normals may differ from
numpy in the last bit of log/cos, which only the benchmark uses).

Workload recipe (the pages' settings where they give them: STEPQuant paper
digest, 方法-1 unit types, widths {2,4,6,8} / {4,6,8}, 32 pivot heads, 512
pivot rows; 方法-3 outlier geometry of about 10x on key rows and 19x on value
columns):
  q ~ N(0,1);  k = n / ||n||, n ~ N(0,1);  v_j ~ gamma_j N(0,1);  beta ~ U(0,1)
  alpha = exp(-ln2 / h), h log-uniform over the workload's half-life range,
          drawn per (layer, head) (GDN) or per (layer, head, key row) (KDA),
          constant over steps and requests
  S_0 = diag(rowscale) G diag(gamma), G ~ N(0,1): one row per head scaled 10x
        and one value column per head scaled 19x (gamma = 19 there, else 1)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

# stream ids
S_Q, S_K, S_V, S_BETA, S_ALPHA, S_G, S_ROWOUT, S_COLOUT = range(1, 9)


def _mix64_int(z: int) -> int:
    z = (z ^ (z >> 30)) * M1 & MASK64
    z = (z ^ (z >> 27)) * M2 & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int, step: int = 0) -> int:
    return _mix64_int(((seed & 0xFFFFFFFF) << 32 ^ (stream & 0xFFFF) << 16 ^ (step & 0xFFFF)
                       ^ (step >> 16) << 48) & MASK64)


def _bits_np(key: int, n: int, start: int = 0) -> np.ndarray:
    idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
        z = z ^ (z >> np.uint64(31))
    return z


def uniform_np(key: int, shape, start: int = 0) -> np.ndarray:
    """Elements start .. start + size - 1 of the stream."""
    n = int(np.prod(shape))
    z = _bits_np(key, n, start)
    return ((z >> np.uint64(11)).astype(np.float64) * 2.0 ** -53).reshape(shape)


def normal_np(key: int, shape, start: int = 0) -> np.ndarray:
    """Elements start .. start + size - 1 of the stream (Box-Muller pairs, so
    start must be even)."""
    assert start % 2 == 0
    n = int(np.prod(shape))
    m = (n + 1) // 2
    z = _bits_np(key, 2 * m, start)
    u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    rad = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * m)
    out[0::2] = rad * np.cos(2.0 * math.pi * u2)
    out[1::2] = rad * np.sin(2.0 * math.pi * u2)
    return out[:n].reshape(shape)


def randint_np(key: int, shape, hi: int) -> np.ndarray:
    n = int(np.prod(shape))
    z = _bits_np(key, n)
    return (z % np.uint64(hi)).astype(np.int64).reshape(shape)


# ---- torch (device) variant of the same integer stream ---------------------

def _to_i64(x: int) -> int:
    return x - (1 << 64) if x >= (1 << 63) else x


def normal_torch(key: int, shape, device, start: int = 0):
    """Same stream as normal_np, evaluated with int64 wrap-around arithmetic."""
    import torch
    n = int(np.prod(shape))
    m = (n + 1) // 2
    idx = torch.arange(start + 1, start + 2 * m + 1, dtype=torch.int64, device=device)

    def srl(x, s):
        return (x >> s) & ((1 << (64 - s)) - 1)

    z = _to_i64(key) + idx * _to_i64(GOLDEN)
    z = (z ^ srl(z, 30)) * _to_i64(M1)
    z = (z ^ srl(z, 27)) * _to_i64(M2)
    z = z ^ srl(z, 31)
    top = srl(z, 11).to(torch.float64)
    u1 = (top[0::2] + 1.0) * 2.0 ** -53
    u2 = top[1::2] * 2.0 ** -53
    rad = torch.sqrt(-2.0 * torch.log(u1))
    out = torch.empty(2 * m, dtype=torch.float64, device=device)
    out[0::2] = rad * torch.cos(2.0 * math.pi * u2)
    out[1::2] = rad * torch.sin(2.0 * math.pi * u2)
    return out[:n].reshape(shape)


def uniform_torch(key: int, shape, device):
    """Same stream as uniform_np, on a device."""
    import torch
    n = int(np.prod(shape))
    idx = torch.arange(1, n + 1, dtype=torch.int64, device=device)

    def srl(x, s):
        return (x >> s) & ((1 << (64 - s)) - 1)

    z = _to_i64(key) + idx * _to_i64(GOLDEN)
    z = (z ^ srl(z, 30)) * _to_i64(M1)
    z = (z ^ srl(z, 27)) * _to_i64(M2)
    z = z ^ srl(z, 31)
    return (srl(z, 11).to(torch.float64) * 2.0 ** -53).reshape(shape)


def initial_states_torch(wl: "Workload", seed: int, n_req: int, layer: int, device):
    """S_0 of one layer, [n_req, 1, H, D, D] float32, on a device (same recipe)."""
    import torch
    gam = torch.from_numpy(column_scales(wl, seed)[layer]).to(device)
    rsc = torch.from_numpy(row_scales(wl, seed)[layer]).to(device)
    G = normal_torch(stream_key(seed, S_G, layer), (n_req, wl.n_heads, wl.d, wl.d), device)
    S = G * rsc[None, :, :, None].double() * gam[None, :, None, :].double()
    return S.float().unsqueeze(1).contiguous()


def step_inputs_torch(wl: "Workload", seed: int, n_req: int, t: int, alpha: np.ndarray, device) -> dict:
    """step_inputs for all layers, generated on a device (same recipe and streams)."""
    import torch
    shape = (n_req, wl.n_layers, wl.n_heads, wl.d)
    q = normal_torch(stream_key(seed, S_Q, t), shape, device)
    n = normal_torch(stream_key(seed, S_K, t), shape, device)
    k = n / torch.sqrt((n * n).sum(dim=-1, keepdim=True))
    gam = torch.from_numpy(column_scales(wl, seed)).to(device).double()
    v = normal_torch(stream_key(seed, S_V, t), shape, device) * gam[None]
    beta = uniform_torch(stream_key(seed, S_BETA, t), (n_req, wl.n_layers, wl.n_heads), device)
    al = torch.from_numpy(np.ascontiguousarray(alpha)).to(device)
    al = al.unsqueeze(0).expand((n_req,) + tuple(al.shape)).contiguous()
    return dict(q=q.float().contiguous(), k=k.float().contiguous(), v=v.float().contiguous(),
                alpha=al.float().contiguous(), beta=beta.float().contiguous())


def _mixed_torch(keys, n: int, device):
    """The integer streams of several keys at once: [len(keys), n] int64
    (the rows of _bits_np for each key, as wrapped int64)."""
    import torch

    def srl(x, s):
        return (x >> s) & ((1 << (64 - s)) - 1)

    k = torch.tensor([_to_i64(int(x)) for x in keys], dtype=torch.int64, device=device)[:, None]
    idx = torch.arange(1, n + 1, dtype=torch.int64, device=device)[None, :]
    z = k + idx * _to_i64(GOLDEN)
    z = (z ^ srl(z, 30)) * _to_i64(M1)
    z = (z ^ srl(z, 27)) * _to_i64(M2)
    return z ^ srl(z, 31)


def _normal_rows_torch(keys, n: int, device):
    """normal_torch(key, (n,)) for every key, stacked: [len(keys), n] float64."""
    import torch
    m = (n + 1) // 2
    z = _mixed_torch(keys, 2 * m, device)
    top = ((z >> 11) & ((1 << 53) - 1)).to(torch.float64)
    u1 = (top[:, 0::2] + 1.0) * 2.0 ** -53
    u2 = top[:, 1::2] * 2.0 ** -53
    rad = torch.sqrt(-2.0 * torch.log(u1))
    out = torch.empty((len(keys), 2 * m), dtype=torch.float64, device=device)
    out[:, 0::2] = rad * torch.cos(2.0 * math.pi * u2)
    out[:, 1::2] = rad * torch.sin(2.0 * math.pi * u2)
    return out[:, :n]


def prompt_inputs_torch(wl: "Workload", seed: int, n_req: int, t0: int, T: int, alpha: np.ndarray, device,
                        lb: int = 0, le: int = None, block: int = 256) -> dict:
    """Tokens t0 .. t0 + T - 1 of step_inputs_torch as one prompt for layers
    [lb, le): q, k, v [n_req, T, le - lb, H, D], beta [n_req, T, le - lb, H],
    alpha [n_req, T, le - lb, H] (per-head gates) or [.., H, D] (per-row gates).
    Generated `block` tokens at a time (same values as one token at a time)."""
    import torch
    le = wl.n_layers if le is None else le
    L, H, D, nL = wl.n_layers, wl.n_heads, wl.d, le - lb
    shape = (n_req, L, H, D)
    out = {k: torch.empty((n_req, T, nL, H, D), dtype=torch.float32, device=device) for k in ("q", "k", "v")}
    al = torch.from_numpy(np.ascontiguousarray(alpha)).to(device).float()[lb:le]   # [nL, H] or [nL, H, D]
    out["alpha"] = torch.empty((n_req, T) + tuple(al.shape), dtype=torch.float32, device=device)
    out["beta"] = torch.empty((n_req, T, nL, H), dtype=torch.float32, device=device)
    gam = torch.from_numpy(column_scales(wl, seed)).to(device).double()[lb:le]
    n_el = int(np.prod(shape))
    for b0 in range(0, T, block):
        ts = list(range(t0 + b0, t0 + min(T, b0 + block)))
        nb = len(ts)

        def gen(stream):
            x = _normal_rows_torch([stream_key(seed, stream, t) for t in ts], n_el, device)
            return x.reshape((nb,) + shape)[:, :, lb:le].transpose(0, 1)   # [n_req, nb, nL, H, D]

        q = gen(S_Q)
        kn = gen(S_K)
        k = kn / torch.sqrt((kn * kn).sum(dim=-1, keepdim=True))
        v = gen(S_V) * gam[None, None]
        zb = _mixed_torch([stream_key(seed, S_BETA, t) for t in ts], n_req * L * H, device)
        beta = (((zb >> 11) & ((1 << 53) - 1)).to(torch.float64) * 2.0 ** -53).reshape(nb, n_req, L, H)
        sl = slice(b0, b0 + nb)
        out["q"][:, sl] = q.float()
        out["k"][:, sl] = k.float()
        out["v"][:, sl] = v.float()
        out["beta"][:, sl] = beta[:, :, lb:le].transpose(0, 1).float()
        out["alpha"][:, sl] = al[None, None].expand((n_req, nb) + tuple(al.shape))
    return out


# ---- workloads -------------------------------------------------------------

@dataclass
class Workload:
    name: str
    mode: int                 # 0 per-head units (GDN), 1 per-key-row units (KDA)
    n_layers: int
    n_heads: int
    d: int
    n_req: int
    steps: int
    bits: tuple
    nominal_bits: float
    n_pivots: int
    halflife: tuple
    seed: int
    calib_seed: int
    calib_req: int = 1
    calib_steps: int = 64
    row_outlier: float = 10.0
    col_outlier: float = 19.0
    horizon: int = 65536
    extra: dict = field(default_factory=dict)

    @property
    def n_units(self):
        return self.n_layers * self.n_heads * (1 if self.mode == 0 else self.d)


def workloads():
    """The workload families (sizes as named; batch sizes are arguments)."""
    return {
        "tiny_gdn": Workload("tiny_gdn", 0, 1, 4, 16, 1, 32, (2, 4, 6), 4.0, 1, (2.0, 500.0), 1001, 2001),
        "qwen_layer": Workload("qwen_layer", 0, 1, 48, 128, 64, 256, (4, 6, 8), 6.0, 1, (4.0, 20000.0),
                               1002, 2002, calib_req=2),
        "qwen_pool6": Workload("qwen_pool6", 0, 48, 48, 128, 70, 64, (4, 6, 8), 6.0, 32, (4.0, 20000.0),
                               1003, 2003, calib_req=1),
        "qwen_pool4": Workload("qwen_pool4", 0, 48, 48, 128, 70, 64, (2, 4, 6, 8), 4.0, 32, (4.0, 20000.0),
                               1003, 2003, calib_req=1),
        "kda_rows": Workload("kda_rows", 1, 20, 32, 128, 128, 128, (4, 6, 8), 6.0, 512, (4.0, 20000.0),
                             1004, 2004, calib_req=1),
        "drift": Workload("drift", 0, 1, 8, 128, 4, 8192, (4, 6, 8), 6.0, 0, (1000.0, 20000.0),
                          1005, 2005, calib_req=2),
        # head dimensions between the tiny and the Qwen-like cases (parity coverage of every
        # compiled d): 2 layers x 8 heads, widths {2,4,6,8}, nominal 5, one pivot head
        "gdn_d32": Workload("gdn_d32", 0, 2, 8, 32, 6, 16, (2, 4, 6, 8), 5.0, 1, (2.0, 2000.0), 1006, 2006),
        "gdn_d64": Workload("gdn_d64", 0, 2, 8, 64, 6, 16, (2, 4, 6, 8), 5.0, 1, (2.0, 2000.0), 1007, 2007),
    }


def gate_halflives(wl: Workload, seed: int) -> np.ndarray:
    """Half-lives, log-uniform; [L, H] (GDN) or [L, H, D] (KDA)."""
    shape = (wl.n_layers, wl.n_heads) if wl.mode == 0 else (wl.n_layers, wl.n_heads, wl.d)
    u = uniform_np(stream_key(seed, S_ALPHA), shape)
    lo, hi = math.log(wl.halflife[0]), math.log(wl.halflife[1])
    return np.exp(lo + (hi - lo) * u)


def gates(wl: Workload, seed: int) -> np.ndarray:
    """alpha = exp(-ln 2 / h) as float32, same shape as gate_halflives."""
    return np.exp(-math.log(2.0) / gate_halflives(wl, seed)).astype(np.float32)


def column_scales(wl: Workload, seed: int) -> np.ndarray:
    """gamma [L, H, D]: 1 except one column per head at col_outlier."""
    g = np.ones((wl.n_layers, wl.n_heads, wl.d), np.float32)
    cols = randint_np(stream_key(seed, S_COLOUT), (wl.n_layers, wl.n_heads), wl.d)
    for l in range(wl.n_layers):
        for h in range(wl.n_heads):
            g[l, h, cols[l, h]] = wl.col_outlier
    return g


def row_scales(wl: Workload, seed: int) -> np.ndarray:
    g = np.ones((wl.n_layers, wl.n_heads, wl.d), np.float32)
    rows = randint_np(stream_key(seed, S_ROWOUT), (wl.n_layers, wl.n_heads), wl.d)
    for l in range(wl.n_layers):
        for h in range(wl.n_heads):
            g[l, h, rows[l, h]] = wl.row_outlier
    return g


def initial_states(wl: Workload, seed: int, n_req: int, layers=None) -> np.ndarray:
    """S_0 [n_req, nL, H, D, D] float32 for the layers in `layers` (default all)."""
    layers = range(wl.n_layers) if layers is None else layers
    gam = column_scales(wl, seed)
    rsc = row_scales(wl, seed)
    out = []
    for l in layers:
        G = normal_np(stream_key(seed, S_G, l), (n_req, wl.n_heads, wl.d, wl.d))
        S = G * rsc[l][None, :, :, None] * gam[l][None, :, None, :]
        out.append(S.astype(np.float32))
    return np.stack(out, axis=1)


def step_inputs(wl: Workload, seed: int, n_req: int, t: int, alpha: np.ndarray = None,
                layers=None) -> dict:
    """Inputs of decode step t: q, k, v [n_req, nL, H, D], alpha, beta."""
    layers = list(range(wl.n_layers) if layers is None else layers)
    L, H, D = wl.n_layers, wl.n_heads, wl.d

    def blocks(gen, key, blk):
        # the (request, layer) blocks of the [n_req, L, ...] stream that are asked for
        return np.stack([np.stack([gen(key, (blk,), start=(r * L + l) * blk) for l in layers])
                         for r in range(n_req)])

    q = blocks(normal_np, stream_key(seed, S_Q, t), H * D).reshape(n_req, len(layers), H, D)
    n = blocks(normal_np, stream_key(seed, S_K, t), H * D).reshape(n_req, len(layers), H, D)
    k = n / np.sqrt((n * n).sum(axis=-1, keepdims=True))
    gam = column_scales(wl, seed)[layers]
    v = blocks(normal_np, stream_key(seed, S_V, t), H * D).reshape(n_req, len(layers), H, D) * gam[None]
    beta = blocks(uniform_np, stream_key(seed, S_BETA, t), H).reshape(n_req, len(layers), H)
    if alpha is None:
        alpha = gates(wl, seed)
    a = alpha[layers]
    al = np.broadcast_to(a[None], (n_req,) + a.shape).copy()
    return dict(q=q.astype(np.float32), k=k.astype(np.float32), v=v.astype(np.float32),
                alpha=al.astype(np.float32), beta=beta.astype(np.float32))
