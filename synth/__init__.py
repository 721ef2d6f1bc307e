"""Seeded synthetic inputs for the neighbor-rebuild path.

This module serves both the CUDA library's tests/benchmark and the oracle's
tests.  It holds none of the method's arithmetic: it draws positions,
species, features and displacement trajectories, and conditions them (see
``cond.c``) so that no pair lies within 1e-4 A of the list radius rc + skin
(where an fp32 distance test could round either way) and no two atoms are
closer than 0.9 A.

The five systems stand in for the workloads of "Ab Initio Accuracy Beyond the
Cutoff" (Tessera), abstract: a uniform random gas, salt solutions of 98k,
1.02M and 10.24M atoms (the last one the size of the live 10.24M-atom salt
solution), and a 10.06M-atom hollow protein-like shell in water (the size of
the Norovirus capsid run).  The real structures and trained model are not
needed for the neighbor path; these systems reproduce the density (0.1
atoms/A^3, 0.12 in the shell), geometry and list lengths.

Recipe (seeded, deterministic):
  * seed = 20261202 + 1000 * cfg + rep; positions from default_rng(seed),
    features from default_rng([seed, 1000000]), step t displacements from
    default_rng([seed, t]).
  * uniform: positions U[0, L)^3, atoms closer than 0.9 A re-drawn.
  * salt: molecule sites chosen at random from a jittered cubic (or 1:1:2)
    lattice (jitter U[-0.25, 0.25] A per axis); rigid 3-site waters (O-H
    0.96 A, H-O-H 104.5 deg, random unit-quaternion orientation), Na and Cl
    on sites of their own; a molecule with an atom closer than 0.9 A to
    another molecule gets a fresh orientation and jitter.
  * capsid: shell atoms uniform in 140 <= r <= 190 A about the box centre at
    0.12 A^-3; waters on lattice sites outside 138 < r < 192 A (2 A gaps at
    both surfaces, the cavity filled); box sized so that the total is
    10.06M atoms.
  * band: an atom in a pair with |d - (rc+skin)| < 1e-4 A gets a fresh
    U[-0.003, 0.003]^3 A nudge (initial frame) or a fresh displacement draw
    (trajectory frames), repeated until no pair is in the band.
  * positions are wrapped in fp64 (x - L floor(x / L)), cast to fp32, and a
    coordinate that rounds to L is set to 0.
  * features N(0, 1) float32 [n, F]; species int8 (O 0, H 1, Na 2, Cl 3,
    shell 4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cond.c")
_LIB = os.path.join(_HERE, "libcond.so")

BAND = 1e-4          # half-width of the forbidden band around rc + skin (A)
DMIN = 0.9           # minimum pair separation (A)
DENSITY = 0.1        # atoms / A^3
SHELL_DENSITY = 0.12
O_H = 0.96
HOH_DEG = 104.5

CONFIGS = {
    1: dict(name="uniform-3k", kind="uniform", n=3000, aspect=(1, 1, 1), rc=6.0, skin=0.5, cap=192, F=8,
            steps=20, sigma=0.02),
    2: dict(name="salt-98k", kind="salt", n_water=32000, n_ion_pairs=1152, aspect=(1, 1, 1), rc=6.0, skin=0.5,
            cap=192, F=32, steps=200, sigma=0.01),
    3: dict(name="salt-1.02M", kind="salt", n_water=333332, n_ion_pairs=12002, aspect=(1, 1, 2), rc=5.75,
            skin=0.5, cap=160, F=64, steps=100, sigma=0.01),
    4: dict(name="salt-10.24M", kind="salt", n_water=3333332, n_ion_pairs=120002, aspect=(1, 1, 1), rc=5.75,
            skin=0.5, cap=160, F=64, steps=50, sigma=0.01),
    5: dict(name="capsid-10.06M", kind="capsid", n_shell=2068444, n_water=2663852, rc=6.0, skin=0.5, cap=224,
            F=64, steps=50, sigma=0.01),
}


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=gnu11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _cond():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L.cond_mark.argtypes = [P, ctypes.c_int64, P, ctypes.c_double, ctypes.c_double, ctypes.c_double, P, P]
        L.cond_mark.restype = ctypes.c_int64
        _lib = L
    return _lib


def mark_forbidden(pos32: np.ndarray, box, r_band: float, dmin: float = DMIN, band: float = BAND):
    """Masks (close, band) of atoms to re-draw (higher index of each pair)."""
    pos32 = np.ascontiguousarray(pos32[:, :3], dtype=np.float32)
    n = len(pos32)
    L = np.ascontiguousarray(np.asarray(box, dtype=np.float64))
    close = np.zeros(n, dtype=np.uint8)
    bandm = np.zeros(n, dtype=np.uint8)
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _cond().cond_mark(P(pos32), n, P(L), float(dmin), float(r_band), float(band), P(close), P(bandm))
    return close.astype(bool), bandm.astype(bool)


def band_clean(pos, box, rs: float, seed: int = 0, max_iter: int = 200) -> np.ndarray:
    """Nudge atoms of hand-made test inputs until no pair lies within BAND of
    rs (the rule every generated input keeps, so that fp32 distances cannot
    flip a list decision).  pos: float32 [n, 3] or [n, 4]; returns a float32
    copy of the same shape.  Non-finite positions are left alone."""
    p = np.array(pos, dtype=np.float32, copy=True)
    rng = np.random.default_rng([seed, 77])
    L32 = np.asarray(box, dtype=np.float32)
    fin = np.isfinite(p[:, :3]).all(1)
    inside = fin & ((p[:, :3] >= 0) & (p[:, :3] < L32)).all(1)
    for _ in range(max_iter):
        q = np.where(fin[:, None], p[:, :3], np.float32(0.0))
        _, bandm = mark_forbidden(q, box, rs, dmin=0.0)
        bandm &= fin
        if not bandm.any():
            return p
        idx = np.nonzero(bandm)[0]
        moved = p[idx, :3].astype(np.float64) + rng.uniform(-0.003, 0.003, size=(len(idx), 3))
        # atoms that were in [0, L) stay there
        ins = inside[idx]
        moved[ins] = wrap_cast(moved[ins], box)
        p[idx, :3] = moved.astype(np.float32)
    raise RuntimeError("band conditioning did not converge")


def wrap_cast(x64: np.ndarray, box) -> np.ndarray:
    """fp64 positions -> fp32 in [0, L): wrap in fp64, cast, fold L to 0."""
    L = np.asarray(box, dtype=np.float64)
    w = x64 - L * np.floor(x64 / L)
    p = w.astype(np.float32)
    L32 = np.asarray(box, dtype=np.float32)
    p = np.where(p >= L32, np.float32(0.0), p)
    return np.ascontiguousarray(p, dtype=np.float32)


def _seed(cfg: int, rep: int) -> int:
    return 20261202 + 1000 * int(cfg) + int(rep)


@dataclass
class System:
    """A generated system: fp32 positions in [0, L), box, parameters."""
    name: str
    pos: np.ndarray            # float32 [n, 3]
    box: tuple                 # three float32 lengths
    rc: float
    skin: float
    cap: int
    F: int
    steps: int
    sigma: float
    seed: int
    species: np.ndarray        # int8 [n]
    pos64: np.ndarray = field(repr=False, default=None)   # unwrapped fp64 positions
    _feat: np.ndarray = field(repr=False, default=None)

    @property
    def n(self) -> int:
        return len(self.pos)

    @property
    def rs(self) -> float:
        return float(np.float32(self.rc) + np.float32(self.skin))

    def features(self) -> np.ndarray:
        if self._feat is None:
            rng = np.random.default_rng([self.seed, 1000000])
            self._feat = rng.standard_normal((self.n, self.F), dtype=np.float32)
        return self._feat

    def pos4(self) -> np.ndarray:
        p = np.zeros((self.n, 4), dtype=np.float32)
        p[:, :3] = self.pos
        return p

    def trajectory(self, steps: int | None = None, condition: bool = True):
        """Yield (t, fp32 positions [n, 3]) for t = 1..steps: a random walk
        of N(0, sigma^2) per axis per step.  With ``condition`` every frame
        is kept free of pairs in the rc+skin band."""
        steps = self.steps if steps is None else steps
        x = self.pos64.copy()
        for t in range(1, steps + 1):
            rng = np.random.default_rng([self.seed, t])
            dx = rng.normal(0.0, self.sigma, size=x.shape)
            p = wrap_cast(x + dx, self.box)
            if condition:
                for _ in range(100):
                    _, bm = mark_forbidden(p, self.box, self.rs, dmin=0.0)
                    if not bm.any():
                        break
                    idx = np.nonzero(bm)[0]
                    dx[idx] = rng.normal(0.0, self.sigma, size=(len(idx), 3))
                    p[idx] = wrap_cast(x[idx] + dx[idx], self.box)
                else:
                    raise RuntimeError("trajectory band conditioning did not converge")
            x = x + dx
            yield t, p


def _box_for(volume: float, aspect) -> tuple:
    a = np.asarray(aspect, dtype=np.float64)
    s = (volume / np.prod(a)) ** (1.0 / 3.0)
    return tuple(float(np.float32(s * ai)) for ai in a)


def _random_rotations(rng, m: int) -> np.ndarray:
    """m random rotation matrices from uniform unit quaternions."""
    q = rng.standard_normal((m, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    w, x, y, z = q.T
    R = np.empty((m, 3, 3))
    R[:, 0, 0] = 1 - 2 * (y * y + z * z); R[:, 0, 1] = 2 * (x * y - z * w); R[:, 0, 2] = 2 * (x * z + y * w)
    R[:, 1, 0] = 2 * (x * y + z * w); R[:, 1, 1] = 1 - 2 * (x * x + z * z); R[:, 1, 2] = 2 * (y * z - x * w)
    R[:, 2, 0] = 2 * (x * z - y * w); R[:, 2, 1] = 2 * (y * z + x * w); R[:, 2, 2] = 1 - 2 * (x * x + y * y)
    return R


def _water_frame() -> np.ndarray:
    h = np.deg2rad(HOH_DEG) / 2.0
    return np.array([[0.0, 0.0, 0.0],
                     [O_H * np.sin(h), O_H * np.cos(h), 0.0],
                     [-O_H * np.sin(h), O_H * np.cos(h), 0.0]])


def _lattice(box, nsites_needed: int, aspect, exclude=None):
    """Smallest lattice of the given aspect with at least nsites_needed sites
    (outside the exclusion test, if given).  Returns site coordinates."""
    a = np.asarray(aspect, dtype=np.int64)
    m = max(1, int(np.floor((nsites_needed / np.prod(a)) ** (1.0 / 3.0))))
    while True:
        dims = m * a
        sp = np.asarray(box, dtype=np.float64) / dims
        g = np.stack(np.meshgrid(*[np.arange(d) for d in dims], indexing="ij"), axis=-1).reshape(-1, 3)
        sites = (g + 0.5) * sp
        if exclude is not None:
            sites = sites[~exclude(sites)]
        if len(sites) >= nsites_needed * 1.005:
            return sites, sp
        m += 1


class _Molecules:
    """Per-molecule bookkeeping so that a molecule can be re-drawn."""

    def __init__(self, sites, kinds, rng, jitter=0.25):
        self.sites = sites            # [m, 3] chosen lattice sites
        self.kinds = kinds            # 0 water, 2 Na, 3 Cl
        self.rng = rng
        self.jitter = jitter
        self.frame = _water_frame()

    def place(self, idx):
        rng = self.rng
        centers = self.sites[idx] + rng.uniform(-self.jitter, self.jitter, size=(len(idx), 3))
        R = _random_rotations(rng, len(idx))
        return centers, R


def _make_salt(cfg_id, c, rep):
    seed = _seed(cfg_id, rep)
    rng = np.random.default_rng(seed)
    n_w, n_p = c["n_water"], c["n_ion_pairs"]
    n_atoms = 3 * n_w + 2 * n_p
    box = _box_for(n_atoms / DENSITY, c["aspect"])
    n_sites = n_w + 2 * n_p
    sites, sp = _lattice(box, n_sites, c["aspect"])
    # a random offset of the whole lattice so that atoms straddle the faces
    sites = sites + rng.uniform(0.0, 1.0, size=3) * sp
    chosen = sites[rng.choice(len(sites), size=n_sites, replace=False)]
    mol_kind = np.concatenate([np.zeros(n_w, np.int8), np.full(n_p, 2, np.int8), np.full(n_p, 3, np.int8)])
    mol = _Molecules(chosen, mol_kind, rng)
    frame = _water_frame()

    # atom layout: waters (O, H, H) first, then Na, then Cl
    atom_mol = np.concatenate([np.repeat(np.arange(n_w), 3), n_w + np.arange(2 * n_p)])
    species = np.concatenate([np.tile(np.array([0, 1, 1], np.int8), n_w), np.full(n_p, 2, np.int8),
                              np.full(n_p, 3, np.int8)])
    x = np.empty((n_atoms, 3))

    def place(mids):
        centers, R = mol.place(mids)
        w = mids < n_w
        wm = mids[w]
        if len(wm):
            pts = centers[w][:, None, :] + np.einsum("mij,kj->mki", R[w], frame)
            base = 3 * wm
            x[base] = pts[:, 0]; x[base + 1] = pts[:, 1]; x[base + 2] = pts[:, 2]
        im = mids[~w]
        if len(im):
            x[3 * n_w + (im - n_w)] = centers[~w]

    place(np.arange(n_sites))
    pos = _condition(x, box, c, rng, redraw_close=lambda bad: place(np.unique(atom_mol[bad])))
    return System(c["name"], pos, box, c["rc"], c["skin"], c["cap"], c["F"], c["steps"], c["sigma"], seed,
                  species, pos64=x)


def _make_uniform(cfg_id, c, rep):
    seed = _seed(cfg_id, rep)
    rng = np.random.default_rng(seed)
    n = c["n"]
    box = _box_for(n / DENSITY, c["aspect"])
    x = rng.uniform(0.0, 1.0, size=(n, 3)) * np.asarray(box)

    def redraw(bad):
        x[bad] = rng.uniform(0.0, 1.0, size=(len(bad), 3)) * np.asarray(box)

    pos = _condition(x, box, c, rng, redraw_close=redraw)
    return System(c["name"], pos, box, c["rc"], c["skin"], c["cap"], c["F"], c["steps"], c["sigma"], seed,
                  np.zeros(n, np.int8), pos64=x)


def _make_capsid(cfg_id, c, rep):
    seed = _seed(cfg_id, rep)
    rng = np.random.default_rng(seed)
    n_s, n_w = c["n_shell"], c["n_water"]
    r_in, r_out, gap = 140.0, 190.0, 2.0
    v_excl = 4.0 / 3.0 * np.pi * ((r_out + gap) ** 3 - (r_in - gap) ** 3)
    Lb = ((3 * n_w) / DENSITY + v_excl) ** (1.0 / 3.0)
    box = _box_for(Lb ** 3, (1, 1, 1))
    ctr = np.asarray(box) / 2.0

    def shell_points(m):
        u = rng.uniform(0.0, 1.0, size=m)
        r = (u * (r_out ** 3 - r_in ** 3) + r_in ** 3) ** (1.0 / 3.0)
        d = rng.standard_normal((m, 3))
        d /= np.linalg.norm(d, axis=1, keepdims=True)
        return ctr + r[:, None] * d

    excl = lambda s: np.abs(np.linalg.norm(s - ctr, axis=1) - (r_in + r_out) / 2.0) < (r_out - r_in) / 2.0 + gap
    sites, sp = _lattice(box, n_w, (1, 1, 1), exclude=excl)
    chosen = sites[rng.choice(len(sites), size=n_w, replace=False)]
    mol = _Molecules(chosen, np.zeros(n_w, np.int8), rng)
    frame = _water_frame()
    n_atoms = n_s + 3 * n_w
    x = np.empty((n_atoms, 3))
    # random sequential addition on the shell alone first: far cheaper than
    # conditioning the whole box while a third of the shell is still close
    xs = shell_points(n_s)
    for _ in range(200):
        close, _ = mark_forbidden(wrap_cast(xs, box), box, r_band=0.0, band=0.0)
        if not close.any():
            break
        bad = np.nonzero(close)[0]
        xs[bad] = shell_points(len(bad))
    x[:n_s] = xs

    def place_w(mids):
        centers, R = mol.place(mids)
        pts = centers[:, None, :] + np.einsum("mij,kj->mki", R, frame)
        base = n_s + 3 * mids
        x[base] = pts[:, 0]; x[base + 1] = pts[:, 1]; x[base + 2] = pts[:, 2]

    place_w(np.arange(n_w))

    def redraw(bad):
        sh = bad[bad < n_s]
        if len(sh):
            x[sh] = shell_points(len(sh))
        wa = bad[bad >= n_s]
        if len(wa):
            place_w(np.unique((wa - n_s) // 3))

    pos = _condition(x, box, c, rng, redraw_close=redraw)
    species = np.concatenate([np.full(n_s, 4, np.int8), np.tile(np.array([0, 1, 1], np.int8), n_w)])
    return System(c["name"], pos, box, c["rc"], c["skin"], c["cap"], c["F"], c["steps"], c["sigma"], seed,
                  species, pos64=x)


def _condition(x, box, c, rng, redraw_close, max_iter=200):
    """Re-draw atoms until no pair is closer than DMIN or within BAND of rs.
    Modifies the fp64 positions x in place; returns the fp32 positions."""
    rs = float(np.float32(c["rc"]) + np.float32(c["skin"]))
    for _ in range(max_iter):
        p = wrap_cast(x, box)
        close, bandm = mark_forbidden(p, box, rs)
        if not close.any() and not bandm.any():
            return p
        if close.any():
            redraw_close(np.nonzero(close)[0])
        idx = np.nonzero(bandm & ~close)[0]
        if len(idx):
            x[idx] += rng.uniform(-0.003, 0.003, size=(len(idx), 3))
    raise RuntimeError("input conditioning did not converge")


_CACHE: dict = {}
_GEN_VERSION = 3   # bump when the recipe changes, so stale disk caches are ignored


def _disk_cache_path(cfg_id: int, rep: int):
    d = os.environ.get("TESS_SYNTH_CACHE", os.path.join("/tmp", "tess_synth_cache"))
    return os.path.join(d, "cfg%d_rep%d_v%d.npz" % (cfg_id, rep, _GEN_VERSION))


def system(cfg_id: int, rep: int = 0, cache: bool = True) -> System:
    """The synthetic system of configuration cfg_id (1..5).  Large systems
    are cached on disk (``$TESS_SYNTH_CACHE``, default /tmp/tess_synth_cache)
    because conditioning 10M atoms takes tens of seconds."""
    key = (cfg_id, rep)
    if cache and key in _CACHE:
        return _CACHE[key]
    c = CONFIGS[cfg_id]
    path = _disk_cache_path(cfg_id, rep)
    s = None
    if cache and os.path.exists(path):
        try:
            z = np.load(path)
            s = System(c["name"], z["pos"], tuple(float(v) for v in z["box"]), c["rc"], c["skin"], c["cap"], c["F"],
                       c["steps"], c["sigma"], _seed(cfg_id, rep), z["species"], pos64=z["pos64"])
        except Exception:
            s = None
    if s is None:
        maker = {"uniform": _make_uniform, "salt": _make_salt, "capsid": _make_capsid}[c["kind"]]
        s = maker(cfg_id, c, rep)
        if cache and s.n >= 500000:
            try:
                os.makedirs(os.path.dirname(path), exist_ok=True)
                tmp = path + ".tmp%d.npz" % os.getpid()
                np.savez(tmp, pos=s.pos, box=np.asarray(s.box, np.float32), species=s.species, pos64=s.pos64)
                os.replace(tmp, path)
            except OSError:
                pass
    if cache:
        _CACHE[key] = s
    return s


def custom(kind: str, size: int, rc: float = 5.75, skin: float = 0.5, cap: int = 160, F: int = 16,
           steps: int = 10, sigma: float = 0.01, aspect=(1, 1, 1), seed_id: int = 90) -> System:
    """A smaller system of the same kind: ``size`` is the atom count for
    'uniform' and the water count for 'salt' (ions at the same 1.17%)."""
    if kind == "uniform":
        c = dict(name="uniform-%d" % size, kind="uniform", n=size, aspect=aspect, rc=rc, skin=skin, cap=cap, F=F,
                 steps=steps, sigma=sigma)
        return _make_uniform(seed_id, c, 0)
    if kind == "salt":
        n_p = max(1, int(round(size * 3 * 0.0117 / 2 / (1 - 0.0117))))
        c = dict(name="salt-%d" % (3 * size + 2 * n_p), kind="salt", n_water=size, n_ion_pairs=n_p, aspect=aspect,
                 rc=rc, skin=skin, cap=cap, F=F, steps=steps, sigma=sigma)
        return _make_salt(seed_id, c, 0)
    raise ValueError(kind)
