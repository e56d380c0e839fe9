"""Seeded synthetic inputs for the edge tensor-product convolution.

The one module that both the CUDA path (tests, bench) and the float64 oracle
use. It draws inputs only -- atom positions, cells, given edge lists, node
features, radial weights and output cotangents -- and holds none of the
method's arithmetic (no neighbour search, harmonics, radial basis, path
enumeration or contraction).

Workloads (shapes of the pages' benchmarks; every number below is part of the
workload description, not of the method):

  tiny      32 atoms uniform in a 6 A non-periodic cube, r_cut 4, 8x0e+8x1o, SH lmax 1
  diamond1k 5x5x5 conventional diamond cells, a = 3.567 A, periodic, jitter N(0, 0.05 A),
            r_cut 5, 64x0e+64x1o+64x2e, SH lmax 2  (the 1000-atom diamond cell of FlashCart Fig. 1)
  sweepL    1024 nodes x exactly 128 edges, senders uniform, directions uniform on S^2,
            lengths U[0.8, 5] A, r_cut 5, 128 channels, lmax L in {1,2,3}, forward only
            (FlashCart Fig. 3a edge-convolution workload)
  diamond8k 10x10x10 cells, jitter N(0, 0.1 A), r_cut 5, 128x(0e,1o,2e,3o), SH lmax 3
  melt32k   32768 atoms, random sequential addition with 1.0 A minimum distance in a periodic
            cube at 0.08 atoms/A^3, r_cut 6, 128x(0e,1o,2e), SH lmax 2

Randomness: numpy PCG64 with independent streams per quantity,
default_rng([seed, k]) with k = 0 positions/edges, 1 node features, 2 radial
weights, 3 output cotangent. Seeds: tiny 1, diamond1k 2, sweepL 30+L,
diamond8k 4, melt32k 5. Features and cotangents ~ N(0, 1); W ~ N(0, 1/8)
(variance 1/n_basis). Everything is returned as float32 (cells float64).
"""
import math
from dataclasses import dataclass

import numpy as np

N_BASIS = 8
A_DIAMOND = 3.567
_DIAMOND_BASIS = np.array([
    [0.0, 0.0, 0.0], [0.0, 0.5, 0.5], [0.5, 0.0, 0.5], [0.5, 0.5, 0.0],
    [0.25, 0.25, 0.25], [0.25, 0.75, 0.75], [0.75, 0.25, 0.75], [0.75, 0.75, 0.25]])


@dataclass
class Workload:
    name: str
    seed: int
    channels: int
    lmax: int               # irreps_in = irreps_out = C x (0e, 1o, 2e, ...) up to lmax; SH lmax = lmax
    r_cut: np.float32
    n_basis: int
    n_nodes: int
    pos: np.ndarray = None       # [N, 3] float32 (None for given-edge workloads)
    cell: np.ndarray = None      # [3, 3] float64 rows = lattice vectors, or None
    pbc: tuple = (False, False, False)
    given_receiver: np.ndarray = None   # given-edge workloads: int64 [E]
    given_sender: np.ndarray = None
    given_edge_vec: np.ndarray = None   # float32 [E, 3]
    forward_only: bool = False

    @property
    def irreps(self):
        return "+".join(f"{self.channels}x{l}{'e' if l % 2 == 0 else 'o'}" for l in range(self.lmax + 1))

    @property
    def dim(self):
        return self.channels * (self.lmax + 1) ** 2

    def rng(self, k):
        return np.random.default_rng([self.seed, k])

    def features(self):
        return self.rng(1).standard_normal((self.n_nodes, self.dim)).astype(np.float32)

    def weights(self, n_paths):
        w = self.rng(2).standard_normal((self.n_basis, n_paths, self.channels)) * math.sqrt(1.0 / 8.0)
        return w.astype(np.float32)

    def cotangent(self):
        return self.rng(3).standard_normal((self.n_nodes, self.dim)).astype(np.float32)


def _wrap(pos, box):
    return np.mod(pos, box)


def _diamond(ncell, jitter, seed, name, channels, lmax, r_cut):
    a = A_DIAMOND
    grid = np.stack(np.meshgrid(np.arange(ncell), np.arange(ncell), np.arange(ncell), indexing="ij"), -1)
    grid = grid.reshape(-1, 3).astype(np.float64)
    pos = (grid[:, None, :] + _DIAMOND_BASIS[None, :, :]).reshape(-1, 3) * a
    box = ncell * a
    rng = np.random.default_rng([seed, 0])
    pos = _wrap(pos + rng.normal(0.0, jitter, size=pos.shape), box)
    return Workload(name=name, seed=seed, channels=channels, lmax=lmax, r_cut=np.float32(r_cut),
                    n_basis=N_BASIS, n_nodes=pos.shape[0], pos=pos.astype(np.float32),
                    cell=np.eye(3) * box, pbc=(True, True, True))


def _tiny(seed=1):
    s = seed
    while True:
        pos = np.random.default_rng([s, 0]).uniform(0.0, 6.0, size=(32, 3))
        diff = pos[:, None, :] - pos[None, :, :]
        dist = np.sqrt((diff ** 2).sum(-1)) + np.eye(32) * 1e9
        if dist.min() >= 0.5:
            break
        s += 1  # documented deterministic re-draw when two atoms are closer than 0.5 A
    return Workload(name="tiny", seed=s, channels=8, lmax=1, r_cut=np.float32(4.0), n_basis=N_BASIS,
                    n_nodes=32, pos=pos.astype(np.float32), cell=None, pbc=(False, False, False))


def _sweep(lmax, n_nodes=1024, degree=128):
    seed = 30 + lmax
    rng = np.random.default_rng([seed, 0])
    n_e = n_nodes * degree
    receiver = np.repeat(np.arange(n_nodes), degree)
    sender = rng.integers(0, n_nodes, size=n_e)
    direc = rng.standard_normal((n_e, 3))
    direc /= np.linalg.norm(direc, axis=1, keepdims=True)
    length = rng.uniform(0.8, 5.0, size=n_e)
    vec = (direc * length[:, None]).astype(np.float32)
    # hand the edges over in a shuffled order: building the CSR is part of the path
    order = rng.permutation(n_e)
    return Workload(name=f"sweep{lmax}", seed=seed, channels=128, lmax=lmax, r_cut=np.float32(5.0),
                    n_basis=N_BASIS, n_nodes=n_nodes, given_receiver=receiver[order].astype(np.int64),
                    given_sender=sender[order].astype(np.int64), given_edge_vec=vec[order],
                    forward_only=True)


def _melt(seed=5, n_atoms=32768, density=0.08, dmin=1.0):
    box = (n_atoms / density) ** (1.0 / 3.0)
    rng = np.random.default_rng([seed, 0])
    ncell = int(box // dmin)
    csize = box / ncell
    grid = {}
    acc = []
    while len(acc) < n_atoms:
        cand = rng.uniform(0.0, box, size=(4096, 3))
        for p in cand:
            c = tuple((p // csize).astype(int) % ncell)
            ok = True
            for dx in (-1, 0, 1):
                for dy in (-1, 0, 1):
                    for dz in (-1, 0, 1):
                        for q in grid.get(((c[0] + dx) % ncell, (c[1] + dy) % ncell, (c[2] + dz) % ncell), ()):
                            d = p - q
                            d -= box * np.round(d / box)
                            if d @ d < dmin * dmin:
                                ok = False
                                break
                        if not ok:
                            break
                    if not ok:
                        break
                if not ok:
                    break
            if ok:
                acc.append(p)
                grid.setdefault(c, []).append(p)
                if len(acc) == n_atoms:
                    break
    pos = np.asarray(acc)
    return Workload(name="melt32k", seed=seed, channels=128, lmax=2, r_cut=np.float32(6.0),
                    n_basis=N_BASIS, n_nodes=n_atoms, pos=pos.astype(np.float32),
                    cell=np.eye(3) * box, pbc=(True, True, True))


def make(name):
    """Build a workload by name: tiny, diamond1k, sweep1, sweep2, sweep3, diamond8k, melt32k."""
    if name == "tiny":
        return _tiny()
    if name == "diamond1k":
        return _diamond(5, 0.05, 2, "diamond1k", 64, 2, 5.0)
    if name.startswith("sweep"):
        return _sweep(int(name[5:]))
    if name == "diamond8k":
        return _diamond(10, 0.1, 4, "diamond8k", 128, 3, 5.0)
    if name == "melt32k":
        return _melt()
    raise KeyError(name)


ALL = ["tiny", "diamond1k", "sweep1", "sweep2", "sweep3", "diamond8k", "melt32k"]
