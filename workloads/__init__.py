"""Seeded synthetic inputs for the five workload shapes.

This module only draws random numbers; it holds none of the quantization
method's arithmetic.  Both the CUDA path and the CPU oracle receive the SAME
bytes produced here (generated once, then copied to wherever they are
needed), so it is the one piece the two sides share.

Recipe (all draws from a seeded ``torch.Generator`` on the target device;
values rounded to bf16 with round-to-nearest-even by ``Tensor.to``):
  * weights: N(0, std); then ``round(p * numel)`` distinct positions, drawn
    uniformly without replacement, are multiplied by the outlier factor;
  * calibration activations: z * c_j with z ~ N(0,1) (or Student-t with 4
    degrees of freedom, z / sqrt(chi2_4 / 4), chi2_4 = -2 ln(U1 U2)) and a
    per-input-channel scale c_j = exp(sigma * N(0,1)) (lognormal);
  * mixture-of-experts routing: every token picks 8 distinct experts by
    Gumbel-top-8 over log p_e with Zipf popularity p_e ~ (e+1)^-1.1; expert e
    gets the rows of the tokens routed to it, stored contiguously in expert
    order (row offsets returned alongside).
These stand in for the model weights and calibration text that the method's
pages use; nothing here reads a dataset.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BF16 = torch.bfloat16


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight(out: int, inp: int, std: float, outlier_frac: float, outlier_mult: float,
           seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    w = torch.empty(out, inp, dtype=torch.float32, device=device)
    w.normal_(0.0, std, generator=g)
    n = w.numel()
    k = int(round(outlier_frac * n))
    if k > 0:
        idx = torch.randperm(n, generator=g, device=device)[:k]
        w.view(-1)[idx] *= outlier_mult
    return w.to(BF16)


def channel_scale(inp: int, sigma: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    z = torch.empty(inp, dtype=torch.float32, device=device).normal_(0.0, 1.0, generator=g)
    return torch.exp(sigma * z)


def calib(tokens: int, inp: int, sigma: float, seed: int, device="cpu", dist: str = "normal",
          chunk_rows: int = 8192, out: torch.Tensor | None = None) -> torch.Tensor:
    """X[tokens, inp] bf16, generated in row chunks to bound temporaries."""
    c = channel_scale(inp, sigma, seed * 1000003 + 17, device)
    g = _gen(seed, device)
    X = out if out is not None else torch.empty(tokens, inp, dtype=BF16, device=device)
    for r0 in range(0, tokens, chunk_rows):
        r1 = min(tokens, r0 + chunk_rows)
        z = torch.empty(r1 - r0, inp, dtype=torch.float32, device=device).normal_(0.0, 1.0, generator=g)
        if dist == "student_t4":
            u1 = 1.0 - torch.rand(r1 - r0, inp, device=device, generator=g)
            u2 = 1.0 - torch.rand(r1 - r0, inp, device=device, generator=g)
            chi2 = -2.0 * torch.log(u1 * u2)
            z = z / torch.sqrt(chi2 / 4.0)
        elif dist != "normal":
            raise ValueError(dist)
        X[r0:r1] = (z * c).to(BF16)
    return X


def moe_routing(tokens: int, experts: int, topk: int, zipf_s: float, seed: int,
                device="cpu", chunk: int = 65536) -> torch.Tensor:
    """Tokens routed to each expert (int64 [experts])."""
    g = _gen(seed, device)
    logp = -zipf_s * torch.log(torch.arange(1, experts + 1, dtype=torch.float32, device=device))
    counts = torch.zeros(experts, dtype=torch.int64, device=device)
    for t0 in range(0, tokens, chunk):
        n = min(chunk, tokens - t0)
        u = torch.rand(n, experts, device=device, generator=g).clamp_min_(1e-20)
        gumbel = -torch.log(-torch.log(u))
        top = torch.topk(logp + gumbel, topk, dim=1).indices
        counts += torch.bincount(top.reshape(-1), minlength=experts)
    return counts


@dataclass
class Matrix:
    name: str
    out: int
    inp: int
    x_key: str                 # which calibration tensor feeds this weight
    seed: int
    std: float
    outlier_frac: float
    outlier_mult: float
    expert: int = -1           # >= 0 for the grouped (MoE) workload: row block of h

    def make(self, device="cpu") -> torch.Tensor:
        return weight(self.out, self.inp, self.std, self.outlier_frac, self.outlier_mult,
                      self.seed, device)


@dataclass
class Calib:
    key: str
    tokens: int
    inp: int
    sigma: float
    seed: int
    dist: str = "normal"
    row_offsets: list[int] | None = None   # MoE: per-expert slices, length experts+1

    def make(self, device="cpu") -> torch.Tensor:
        if self.row_offsets is None:
            return calib(self.tokens, self.inp, self.sigma, self.seed, device, self.dist)
        # grouped: every expert slice has its own channel scales and stream
        X = torch.empty(self.tokens, self.inp, dtype=BF16, device=device)
        for e in range(len(self.row_offsets) - 1):
            r0, r1 = self.row_offsets[e], self.row_offsets[e + 1]
            if r1 > r0:
                calib(r1 - r0, self.inp, self.sigma, self.seed * 4099 + e, device, self.dist,
                      out=X[r0:r1])
        return X


@dataclass
class Run:
    lo: int
    hi: int
    weighted: bool             # False: plain MSE (h == 1)


@dataclass
class Workload:
    name: str
    q_max: float
    matrices: list[Matrix]
    calibs: dict[str, Calib]
    runs: list[Run]
    experts: int = 0
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def weight_elems(self) -> int:
        return sum(m.out * m.inp for m in self.matrices)

    @property
    def calib_bytes(self) -> int:
        return sum(c.tokens * c.inp * 2 for c in self.calibs.values())


def single_layer() -> Workload:
    """W 256x1024 N(0,0.02), 0.5% x10 outliers; X 512x1024 N(0,1)*lognormal(1)."""
    return Workload(
        "single_layer_256x1024", 448.0,
        [Matrix("w", 256, 1024, "x", 101, 0.02, 0.005, 10.0)],
        {"x": Calib("x", 512, 1024, 1.0, 1)},
        [Run(-9, 6, True)])


def square_layer() -> Workload:
    """W 4096x4096 N(0,0.02), 0.1% x8; X 8192x4096 Student-t(4)*lognormal(1); Q=256;
    MSE [-3,+7] and WMSE [-8,+7]."""
    return Workload(
        "square_4096x4096", 256.0,
        [Matrix("w", 4096, 4096, "x", 202, 0.02, 0.001, 8.0)],
        {"x": Calib("x", 8192, 4096, 1.0, 2, "student_t4")},
        [Run(-3, 7, False), Run(-8, 7, True)])


def llama3_8b() -> Workload:
    """Llama-3-8B-shaped projections; X 16384 tokens per input site."""
    m = [("q", 4096, 4096, "attn"), ("k", 1024, 4096, "attn"), ("v", 1024, 4096, "attn"),
         ("o", 4096, 4096, "o"), ("gate", 14336, 4096, "mlp"), ("up", 14336, 4096, "mlp"),
         ("down", 4096, 14336, "down")]
    mats = [Matrix(n, o, i, x, 300 + k, 0.02, 0.001, 10.0) for k, (n, o, i, x) in enumerate(m)]
    cal = {"attn": Calib("attn", 16384, 4096, 1.0, 31), "o": Calib("o", 16384, 4096, 1.0, 32),
           "mlp": Calib("mlp", 16384, 4096, 1.0, 33), "down": Calib("down", 16384, 14336, 1.0, 34)}
    return Workload("llama3_8b_projections", 448.0, mats, cal, [Run(-9, 6, True)])


def llama33_70b_mlp(seed_offset: int = 0) -> Workload:
    """Llama-3.3-70B-shaped MLP: gate/up 28672x8192, down 8192x28672, N(0,0.015),
    0.1% x10; X 65536 tokens, lognormal(1.5) channel scales."""
    s = 400 + 97 * seed_offset
    mats = [Matrix("gate", 28672, 8192, "gu", s + 1, 0.015, 0.001, 10.0),
            Matrix("up", 28672, 8192, "gu", s + 2, 0.015, 0.001, 10.0),
            Matrix("down", 8192, 28672, "down", s + 3, 0.015, 0.001, 10.0)]
    cal = {"gu": Calib("gu", 65536, 8192, 1.5, s + 41),
           "down": Calib("down", 65536, 28672, 1.5, s + 42)}
    return Workload("llama33_70b_mlp", 448.0, mats, cal, [Run(-9, 6, True)])


def llama33_70b_mlp_x2(seed_offset: int = 0, layers: int = 2) -> Workload:
    """Consecutive Llama-3.3-70B-shaped MLP layers, quantized in one call: layer
    0 is llama33_70b_mlp (same seeds), each further layer its own draw."""
    mats, cal, groups = [], {}, []
    for l in range(layers):
        one = llama33_70b_mlp(seed_offset) if l == 0 else llama33_70b_mlp(seed_offset + 1000 * l)
        groups.append([])
        for m in one.matrices:
            mats.append(Matrix(f"L{l}.{m.name}", m.out, m.inp, f"L{l}.{m.x_key}", m.seed, m.std,
                               m.outlier_frac, m.outlier_mult))
            groups[-1].append(mats[-1].name)
        for k, c in one.calibs.items():
            cal[f"L{l}.{k}"] = Calib(f"L{l}.{k}", c.tokens, c.inp, c.sigma, c.seed, c.dist)
    return Workload(f"llama33_70b_mlp_x{layers}", 448.0, mats, cal, [Run(-9, 6, True)],
                    extra={"layers": groups})


def mlp_layer_slice(seed_offset: int = 0) -> Workload:
    """A whole 70B-MLP-like layer at profiling size: gate/up 8192x4096, down
    4096x8192, N(0,0.015), 0.1% x10; X 16384 tokens x {4096, 8192},
    lognormal(1.5) channel scales (inputs larger than L2)."""
    s = 800 + 97 * seed_offset
    mats = [Matrix("gate", 8192, 4096, "gu", s + 1, 0.015, 0.001, 10.0),
            Matrix("up", 8192, 4096, "gu", s + 2, 0.015, 0.001, 10.0),
            Matrix("down", 4096, 8192, "down", s + 3, 0.015, 0.001, 10.0)]
    cal = {"gu": Calib("gu", 16384, 4096, 1.5, s + 41),
           "down": Calib("down", 16384, 8192, 1.5, s + 42)}
    return Workload("mlp_layer_slice", 448.0, mats, cal, [Run(-9, 6, True)])


def mlp_slice(seed_offset: int = 0) -> Workload:
    """One 70B-MLP-like layer at profiling size: W 8192x8192 N(0,0.015), 0.1% x10;
    X 16384 x 8192, lognormal(1.5) channel scales (inputs larger than L2)."""
    s = 700 + 97 * seed_offset
    return Workload("mlp_slice_8192x8192", 448.0,
                    [Matrix("w", 8192, 8192, "x", s + 1, 0.015, 0.001, 10.0)],
                    {"x": Calib("x", 16384, 8192, 1.5, s + 41)}, [Run(-9, 6, True)])


def moe_grouped(tokens: int = 262144, experts: int = 128, device="cpu") -> Workload:
    """128 experts x {gate, up 768x2048; down 2048x768}; 262144 tokens routed
    top-8 with Zipf(1.1) popularity; per-expert X slices and h."""
    counts = moe_routing(tokens, experts, 8, 1.1, 5, device).cpu().tolist()
    offs = [0]
    for c in counts:
        offs.append(offs[-1] + int(c))
    mats = []
    for e in range(experts):
        mats.append(Matrix(f"e{e}.gate", 768, 2048, "gu", 5000 + 3 * e, 0.02, 0.001, 10.0, e))
        mats.append(Matrix(f"e{e}.up", 768, 2048, "gu", 5001 + 3 * e, 0.02, 0.001, 10.0, e))
        mats.append(Matrix(f"e{e}.down", 2048, 768, "down", 5002 + 3 * e, 0.02, 0.001, 10.0, e))
    cal = {"gu": Calib("gu", offs[-1], 2048, 1.0, 51, row_offsets=offs),
           "down": Calib("down", offs[-1], 768, 1.0, 52, row_offsets=offs)}
    return Workload("moe_128x_gate_up_768x2048_down_2048x768", 448.0, mats, cal,
                    [Run(-9, 6, True)], experts=experts)


ALL = {"single_layer": single_layer, "square_layer": square_layer, "llama3_8b": llama3_8b,
       "llama33_70b_mlp": llama33_70b_mlp, "mlp_slice": mlp_slice, "moe_grouped": moe_grouped,
       "mlp_layer_slice": mlp_layer_slice, "llama33_70b_mlp_x2": llama33_70b_mlp_x2}
