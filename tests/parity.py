"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle, compare.

Tolerance for attention outputs (fp16 / bf16 inputs): max |gpu - oracle| <= 2e-3
and, per (sequence, head), ||gpu - oracle||_inf / ||oracle||_inf <= 1e-2.  The
output is rounded to the storage dtype at the end, and even an exact kernel is
half an ulp of that dtype away from the fp64 oracle, so half an ulp of
|oracle| is allowed on top of both bounds.  For fp32 inputs the path computes
in fp32 throughout: 1e-5 absolute, 1e-4 relative.
"""

from __future__ import annotations

import numpy as np

from oracle import c_oracle
from oracle import reference as R

TOL = {"f16": (2e-3, 1e-2), "bf16": (2e-3, 1e-2), "f32": (1e-5, 1e-4)}
ULP_HALF = {"f16": 2.0 ** -11, "bf16": 2.0 ** -8, "f32": 0.0}   # half an ulp, relative


def torch_dtype(dtype: str):
    import torch

    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def to_device(arr: np.ndarray, dtype: str | None, device="cuda"):
    """Host array (bf16 as uint16 bits) -> torch tensor on the device."""
    import torch

    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def to_host(t, dtype: str) -> np.ndarray:
    """Device tensor -> host array in the oracle's storage convention."""
    import torch

    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def out_f64(t) -> np.ndarray:
    import torch

    return t.to(torch.float64).cpu().numpy()


def compare(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    """Assert the attention tolerance; return (max_abs, max_rel) without the rounding allowance."""
    atol, rtol = TOL[dtype]
    gpu = np.asarray(gpu, dtype=np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    allow = ULP_HALF[dtype] * np.abs(ref)
    bad = err > atol + allow
    assert not bad.any(), f"{what}: abs error {err.max():.3e} at {np.argwhere(bad)[:3].tolist()}"
    rown = np.abs(ref).max(axis=1)
    rowe = err.max(axis=1)
    rowallow = (ULP_HALF[dtype] * np.abs(ref)).max(axis=1)
    zero_rows = rown == 0
    assert (rowe[zero_rows] == 0).all(), f"{what}: rows that must be zero are not"
    nz = ~zero_rows
    rel = np.zeros_like(rown)
    rel[nz] = np.maximum(rowe[nz] - rowallow[nz], 0) / rown[nz]
    assert (rel <= rtol).all(), f"{what}: rel error {rel.max():.3e}"
    raw_rel = float((rowe[nz] / rown[nz]).max()) if nz.any() else 0.0
    return float(err.max()), raw_rel


def round_to_storage_bits(ref: np.ndarray, dtype: str) -> np.ndarray:
    """The fp64 oracle rounded to the storage dtype, round-to-nearest-even, as raw uint16 bits.

    f16 uses NumPy's conversion (correctly rounded from float64).  bf16 takes the
    candidate from float32 and its two neighbours and keeps the nearest in fp64
    (ties to the even pattern), so no double rounding creeps in.
    """
    ref = np.asarray(ref, dtype=np.float64)
    if dtype == "f16":
        return ref.astype(np.float16).view(np.uint16)
    assert dtype == "bf16"
    b32 = ref.astype(np.float32).view(np.uint32).astype(np.int64)
    cand = (b32 + 0x7FFF + ((b32 >> 16) & 1)) >> 16
    best, best_err = cand.copy(), None
    for d in (-1, 0, 1):
        c = (cand + d) & 0xFFFF
        v = (c.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        err = np.abs(v - ref)
        if best_err is None:
            best, best_err = c, err
        else:
            take = (err < best_err) | ((err == best_err) & ((c & 1) == 0))
            best = np.where(take, c, best)
            best_err = np.where(take, err, best_err)
    return best.astype(np.uint16)


def _ordered(bits: np.ndarray) -> np.ndarray:
    """16-bit sign-magnitude patterns -> integers in value order (adjacent values differ by 1)."""
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def ulp_distance(gpu_bits: np.ndarray, ref: np.ndarray, dtype: str) -> np.ndarray:
    """How many representable steps of the storage dtype lie between the GPU output and RNE(oracle)."""
    return np.abs(_ordered(np.asarray(gpu_bits).view(np.uint16)) - _ordered(round_to_storage_bits(ref, dtype)))


def abs_values(arr: np.ndarray, dtype: str) -> np.ndarray:
    """|x| of a host array in the oracle's storage convention (bf16 as uint16 bits)."""
    return (arr & np.uint16(0x7FFF)) if dtype == "bf16" else np.abs(arr)


# Sharper checks than the tolerance (16-bit outputs), next to compare().
#
# bf16: the decode kernel carries P as a hi + lo pair of bf16 (about 16
# significant bits), so beyond fp32 rounding the only error is the final
# rounding to bf16.  Every element must be within 1 representable step of the
# oracle rounded to bf16 (round-to-nearest-even), unless its absolute error is
# below 2^-20 (outputs near zero, where a step is far smaller than the fp32
# accumulation error).
#
# f16: the decode kernel rounds each p to f16 (relative error <= 2^-11) before
# the PV product and sums l from the unrounded p, so
#     |out - oracle| <= 2^-11 * sum_i p_i |v_i| / sum_i p_i   (P rounding)
#                     + 2^-11 * |oracle|                      (output rounding)
# where the first sum is the oracle's own result with |V| in place of V.
# Every element must meet that bound (times 1.01, plus 2^-16 for fp32
# accumulation and f16 subnormal p); its rows with few comparable keys reach
# several output steps, so a step count is reported, not asserted.
BF16_FLOOR = 2.0 ** -20


def sharp_check(gpu_t, ref: np.ndarray, dtype: str, ref_absv: np.ndarray | None = None, what: str = "") -> dict:
    """Assert the check above for a device tensor of 16-bit outputs; return its statistics."""
    import torch

    if dtype not in ("bf16", "f16"):
        return {}
    gbits = gpu_t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(ref.shape)
    gval = gpu_t.to(torch.float64).cpu().numpy().reshape(ref.shape)
    dist = ulp_distance(gbits, ref, dtype)
    err = np.abs(gval - ref)
    if dtype == "bf16":
        bad = (dist > 1) & (err > BF16_FLOOR)
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond 1 step of RNE(oracle), "
                               f"max {int(dist[bad].max())} steps, abs error {float(err[bad].max()):.3e}")
        worst = None
    else:
        assert ref_absv is not None
        bound = 1.01 * 2.0 ** -11 * (ref_absv.reshape(ref.shape) + np.abs(ref)) + 2.0 ** -16
        bad = err > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the P-rounding bound, "
                               f"worst error/bound {float((err / bound).max()):.3f}")
        worst = float((err / bound).max())
    return {"max_abs": float(err.max()), "over_2e-3": int((err > 2e-3).sum()), "max_steps": int(dist.max()),
            "within_1_step": float((dist <= 1).mean()), "worst_err_over_bound": worst, "elements": int(dist.size)}


class DeviceCase:
    """A workload's tensors on the device plus host copies taken before any kernel ran."""

    def __init__(self, wl, vals_host=None, device_draw=False, device="cuda"):
        import torch

        self.wl = wl
        c = wl.cfg
        self.dtype = c.dtype
        if device_draw:
            from workloads import device_values

            self.dev = device_values(wl, device)
        else:
            from workloads import host_values

            vh = vals_host if vals_host is not None else host_values(wl)
            self.dev = {k: to_device(v, c.dtype, device) for k, v in vh.items()}
        self.block_tables = torch.from_numpy(wl.block_tables).to(device)
        self.context_lens = torch.from_numpy(wl.context_lens).to(device)
        self.slot_mapping = torch.from_numpy(wl.slot_mapping).to(device)
        self.copy_pairs = torch.from_numpy(np.ascontiguousarray(wl.copy_pairs)).to(device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def poison_unread(self):
        """NaN into every pool slot no sequence reads (the tails of last blocks, unused blocks)."""
        import torch

        from workloads import unread_slots

        blk, off = unread_slots(self.wl)
        dev = self.dev["key_cache"].device
        bi = torch.from_numpy(blk).to(dev)
        oi = torch.from_numpy(off).to(dev)
        for k in ("key_cache", "value_cache"):
            self.dev[k][bi, :, oi, :] = float("nan")
        return int(blk.size)

    def host_subproblem(self, seqs):
        """Compact host copy (pre-step) of everything the oracle needs for sequences ``seqs``.

        Blocks the sequences use -- plus copy-pair sources feeding them -- are
        copied off the device and renumbered 0..n-1.
        """
        import torch

        wl = self.wl
        bs = wl.cfg.block_size
        seqs = list(seqs)
        nblk = [-(-int(wl.context_lens[b]) // bs) for b in seqs]
        used = set()
        for b, n in zip(seqs, nblk):
            used.update(int(x) for x in wl.block_tables[b, :n])
        pairs = [(int(s), int(d)) for s, d in wl.copy_pairs if int(d) in used]
        used.update(s for s, _ in pairs)
        ids = sorted(used)
        remap = {old: new for new, old in enumerate(ids)}
        idx = torch.tensor(ids, dtype=torch.long, device=self.dev["key_cache"].device)
        kc = to_host(self.dev["key_cache"].index_select(0, idx), self.dtype)
        vc = to_host(self.dev["value_cache"].index_select(0, idx), self.dtype)
        bt = np.full((len(seqs), max(1, max(nblk))), -1, dtype=np.int32)
        for i, (b, n) in enumerate(zip(seqs, nblk)):
            bt[i, :n] = [remap[int(x)] for x in wl.block_tables[b, :n]]
        # appended tokens of these sequences (slot_mapping row b <-> sequence b for unpadded workloads)
        keys, vals, slots = [], [], []
        key_h = to_host(self.dev["key"], self.dtype)
        val_h = to_host(self.dev["value"], self.dtype)
        real = np.flatnonzero(wl.slot_mapping >= 0)
        for b in seqs:
            t = real[b]
            s = int(wl.slot_mapping[t])
            keys.append(key_h[t])
            vals.append(val_h[t])
            slots.append(remap[s // bs] * bs + s % bs)
        q = to_host(self.dev["q"], self.dtype)[seqs]
        return dict(q=q, key_cache=kc, value_cache=vc, block_tables=bt,
                    context_lens=wl.context_lens[seqs].copy(),
                    key=np.stack(keys), value=np.stack(vals), slot_mapping=np.asarray(slots, np.int64),
                    copy_pairs=np.asarray([(remap[s], remap[d]) for s, d in pairs], np.int64).reshape(-1, 2))


def oracle_step(sub, cfg, do_copy=True, do_write=True):
    """Oracle for one step on a host subproblem: copy-on-write, append, then decode (fp64)."""
    kc, vc = sub["key_cache"], sub["value_cache"]
    if do_copy and len(sub["copy_pairs"]):
        kc, vc = R.copy_blocks(kc, vc, sub["copy_pairs"])
    if do_write:
        kc, vc = R.reshape_and_cache(sub["key"], sub["value"], kc, vc, sub["slot_mapping"])
    return c_oracle.decode(sub["q"], kc, vc, sub["block_tables"], sub["context_lens"], cfg.scale, cfg.dtype,
                           cfg.num_kv_heads)
