"""Seeded synthetic inputs shaped like the workloads on the pages.

This module is shared by the tests, the benchmark and the oracle-side checks.
It draws random numbers and nothing else: no quantization, no scale, no
observer and no other step of the method lives here.

Every tensor comes from its own ``torch.Generator`` seeded with
``seed(config, layer, role)``.  The same call on the same device always returns
the same values; a CUDA generator and a CPU generator give different values, so
a test that checks the CUDA path against the oracle draws once and hands the
same tensor to both sides.

Workloads (sizes and distributions):

* ``c0`` tiny gated MLP: M=64, d=256, I=704.  X ~ N(0,1) in BF16 with 4 outlier
  channels (indices drawn from the seed) scaled x20.  Wg, Wu ~ N(0,0.02) [I,d],
  Wd ~ N(0,0.02) [d,I].  16 calibration batches of the same distribution.
* ``c1`` single Linear sweep: M in {256,1024,4096}, K=2048, N in {2048,8192}.
  X ~ Student-t(nu=4) at unit scale, W ~ N(0,0.02).
* ``c2`` two-input SwiGLU sweep: G ~ N(0, std 2), U ~ N(0,1), [M,I] with
  M in {1024,4096,16384}, I in {8192,11008,14336}.
* ``c3`` shared-quant attention projections: X [2048,3072] ~ N(0,1) with 4
  outlier channels drawn Student-t(nu=4) x20; Wq [3072,3072], Wk, Wv [1024,3072]
  ~ N(0,0.02).
* ``c4`` two-tower decoder MLP pass: 36 layers x {understanding M=1024,
  generation M=4096}, d=3072, I=12288, the c0 distributions, one seed per
  layer and tower.
"""

from __future__ import annotations

import torch

# Role numbers: one per distinct random tensor of a layer.  Calibration batch b
# uses role CALIB + b, so roles stay below 1000 and seeds never collide.
ROLE = {
    "x": 0, "wg": 1, "wu": 2, "wd": 3, "wq": 4, "wk": 5, "wv": 6,
    "g": 7, "u": 8, "outlier": 9, "w": 10,
}
CALIB = 100
N_CALIB = 16

C0 = dict(M=64, d=256, I=704)
C1_M = (256, 1024, 4096)
C1_N = (2048, 8192)
C1_K = 2048
C2_M = (1024, 4096, 16384)
C2_I = (8192, 11008, 14336)
C3 = dict(M=2048, d=3072, Nq=3072, Nk=1024, Nv=1024)
C4 = dict(layers=36, M_und=1024, M_gen=4096, d=3072, I=12288)
W_STD = 0.02
OUTLIER_CHANNELS = 4
OUTLIER_GAIN = 20.0


def seed(config: int, layer: int = 0, role: int = 0) -> int:
    """Seed of one tensor: 1_000_000*config + 1000*layer + role (role < 1000)."""
    if not 0 <= role < 1000:
        raise ValueError("role must be in [0, 1000)")
    return 1_000_000 * config + 1000 * layer + role


def _gen(s: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def normal(shape, std: float, s: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and stored as BF16."""
    g = _gen(s, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def student_t(shape, nu: int, s: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """Student-t with integer nu at unit scale: z / sqrt(chi2_nu / nu), with
    chi2_nu the sum of nu squared standard normals."""
    g = _gen(s, device)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        e = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(e, e)
    return (z / torch.sqrt(chi2 / nu)).to(dtype)


def outlier_channels(d: int, s: int) -> torch.Tensor:
    """Indices of the outlier channels of a layer (drawn on the CPU so that
    every device picks the same channels)."""
    g = _gen(s, "cpu")
    return torch.randperm(d, generator=g)[:OUTLIER_CHANNELS].sort().values


def activation_with_outliers(M: int, d: int, config: int, layer: int, role: int,
                             device="cpu", heavy_tailed_outliers: bool = False) -> torch.Tensor:
    """X ~ N(0,1) [M,d] in BF16 with OUTLIER_CHANNELS channels scaled by
    OUTLIER_GAIN.  With heavy_tailed_outliers the outlier channels are drawn
    Student-t(nu=4) before the gain.  The channel indices depend on (config,
    layer) only, so the evaluation input and the calibration batches of a layer
    share them."""
    s = seed(config, layer, role)
    g = _gen(s, device)
    x = torch.randn((M, d), generator=g, device=device, dtype=torch.float32)
    ch = outlier_channels(d, seed(config, layer, ROLE["outlier"])).to(device)
    if heavy_tailed_outliers:
        t = student_t((M, OUTLIER_CHANNELS), 4, s + 500_000, device, torch.float32)
        x[:, ch] = t
    x[:, ch] *= OUTLIER_GAIN
    return x.to(torch.bfloat16)


def calib_role(b: int) -> int:
    return CALIB + b


# ---------------------------------------------------------------- workloads


def c0_mlp(device="cpu"):
    """Tiny gated MLP: X, Wg, Wu, Wd and 16 calibration batches."""
    M, d, I = C0["M"], C0["d"], C0["I"]
    x = activation_with_outliers(M, d, 0, 0, ROLE["x"], device)
    calib = [activation_with_outliers(M, d, 0, 0, calib_role(b), device) for b in range(N_CALIB)]
    wg = normal((I, d), W_STD, seed(0, 0, ROLE["wg"]), device)
    wu = normal((I, d), W_STD, seed(0, 0, ROLE["wu"]), device)
    wd = normal((d, I), W_STD, seed(0, 0, ROLE["wd"]), device)
    return dict(x=x, calib=calib, wg=wg, wu=wu, wd=wd)


def c1_linear(M: int, N: int, device="cpu", n_calib: int = N_CALIB, calib_rows: int | None = None):
    """Single Linear: X ~ Student-t(4) [M,K], W ~ N(0,0.02) [N,K] and calibration
    batches of calib_rows rows (default M)."""
    K = C1_K
    layer = C1_M.index(M) * 10 + C1_N.index(N) if (M in C1_M and N in C1_N) else 99
    x = student_t((M, K), 4, seed(1, layer, ROLE["x"]), device)
    w = normal((N, K), W_STD, seed(1, layer, ROLE["w"]), device)
    r = M if calib_rows is None else calib_rows
    calib = [student_t((r, K), 4, seed(1, layer, calib_role(b)), device) for b in range(n_calib)]
    return dict(x=x, w=w, calib=calib)


def c2_swiglu(M: int, I: int, device="cpu", n_calib: int = N_CALIB, calib_rows: int | None = None):
    """Two-input SwiGLU: G ~ N(0, std 2), U ~ N(0,1) [M,I] and calibration
    batches (G_b, U_b) of calib_rows rows (default M)."""
    layer = C2_M.index(M) * 10 + C2_I.index(I) if (M in C2_M and I in C2_I) else 99
    g = normal((M, I), 2.0, seed(2, layer, ROLE["g"]), device)
    u = normal((M, I), 1.0, seed(2, layer, ROLE["u"]), device)
    r = M if calib_rows is None else calib_rows
    calib = [(normal((r, I), 2.0, seed(2, layer, calib_role(b)), device),
              normal((r, I), 1.0, seed(2, layer, calib_role(b) + 400), device))
             for b in range(n_calib)]
    return dict(g=g, u=u, calib=calib)


def c3_qkv(device="cpu", n_calib: int = N_CALIB, calib_rows: int | None = None):
    """Shared-quant attention projections."""
    M, d = C3["M"], C3["d"]
    x = activation_with_outliers(M, d, 3, 0, ROLE["x"], device, heavy_tailed_outliers=True)
    r = M if calib_rows is None else calib_rows
    calib = [activation_with_outliers(r, d, 3, 0, calib_role(b), device, heavy_tailed_outliers=True)
             for b in range(n_calib)]
    wq = normal((C3["Nq"], d), W_STD, seed(3, 0, ROLE["wq"]), device)
    wk = normal((C3["Nk"], d), W_STD, seed(3, 0, ROLE["wk"]), device)
    wv = normal((C3["Nv"], d), W_STD, seed(3, 0, ROLE["wv"]), device)
    return dict(x=x, calib=calib, wq=wq, wk=wk, wv=wv)


def c4_layer(layer: int, tower: str, device="cpu", with_x: bool = True,
             n_calib: int = N_CALIB, calib_rows: int | None = None):
    """One tower of one decoder layer of the two-tower pass.  Tower 'und' has
    M=1024 tokens and 'gen' M=4096.  Layer index l and tower t map to seed
    layer 2*l + (t == 'gen')."""
    if tower not in ("und", "gen"):
        raise ValueError(tower)
    M = C4["M_und"] if tower == "und" else C4["M_gen"]
    d, I = C4["d"], C4["I"]
    sl = 2 * layer + (tower == "gen")
    out = dict(M=M)
    out["wg"] = normal((I, d), W_STD, seed(4, sl, ROLE["wg"]), device)
    out["wu"] = normal((I, d), W_STD, seed(4, sl, ROLE["wu"]), device)
    out["wd"] = normal((d, I), W_STD, seed(4, sl, ROLE["wd"]), device)
    if with_x:
        out["x"] = activation_with_outliers(M, d, 4, sl, ROLE["x"], device)
    if n_calib:
        r = M if calib_rows is None else calib_rows
        out["calib"] = [activation_with_outliers(r, d, 4, sl, calib_role(b), device)
                        for b in range(n_calib)]
    return out
