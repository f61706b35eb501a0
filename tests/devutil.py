"""Moves workloads.Problem instances to the GPU with guard bands, runs the
library through its C ABI binding, and checks write sets.

Every device tensor sits inside a larger buffer: `GUARD` canary elements
before and after, plus `misalign` extra elements so that the tensor can start
off a 16-byte boundary.  After a call the guards must be bit-identical.
"""
import numpy as np
import torch

from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import Problem

GUARD = 64  # elements (128 bytes: keeps the base alignment of the allocation)
CANARY = 0x5A5A
SENTINEL = 0x7FFF  # NaN in bf16 and fp16


def tdtype(p: Problem):
    return torch.bfloat16 if p.dtype == "bf16" else torch.float16


class Guarded:
    """A 2-D or 3-D uint16 tensor in a canary-guarded flat device buffer."""

    def __init__(self, bits: np.ndarray, dtype, misalign: int = 0, device="cuda"):
        self.shape = bits.shape
        n = bits.size
        self.lead = GUARD + misalign
        host = np.full(self.lead + n + GUARD, CANARY, dtype=np.uint16)
        host[self.lead: self.lead + n] = bits.ravel()
        self.buf = torch.from_numpy(host.view(np.int16)).to(device)
        self.n = n
        self.t = self.buf[self.lead: self.lead + n].view(dtype).view(*bits.shape)

    def guards_intact(self) -> bool:
        h = self.buf.cpu().numpy().view(np.uint16)
        return bool((h[: self.lead] == CANARY).all() and (h[self.lead + self.n:] == CANARY).all())

    def bits(self) -> np.ndarray:
        return self.t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(self.shape)


def tables(p: Problem, device="cuda", identity=False):
    si = torch.from_numpy(p.seg_indptr.astype(np.int32)).to(device)
    wi = torch.from_numpy(p.weight_indices.astype(np.int32)).to(device)
    pm = None if identity else torch.from_numpy(p.permutation.astype(np.int32)).to(device)
    return si, wi, pm


def run_shrink(p: Problem, workspace: bool = True, out_fill=SENTINEL, identity=False,
               stream=None):
    """Returns (out_r bits [tok, S*rs], guards_ok)."""
    dt = tdtype(p)
    x = Guarded(p.x, dt, p.misalign)
    A = Guarded(p.A, dt, p.misalign)
    out = Guarded(np.full((p.tok, p.S * p.rs), out_fill, dtype=np.uint16), dt, p.misalign)
    si, wi, pm = tables(p, identity=identity)
    ws = lora.make_workspace(p.tok, p.nseg, p.L) if workspace else None
    lora.lora_shrink(x.t[:, : p.K], A.t, si, wi, pm, out.t, num_slices=p.S, rank=p.r,
                     workspace=ws, stream=stream)
    torch.cuda.synchronize()
    ok = x.guards_intact() and A.guards_intact() and out.guards_intact()
    return out.bits(), ok


def run_expand(p: Problem, in_r_bits=None, workspace: bool = True, identity=False,
               scalings=None, stream=None):
    """Returns (base bits [tok, ld_base], guards_ok)."""
    dt = tdtype(p)
    in_r = Guarded(p.in_r if in_r_bits is None else in_r_bits, dt, p.misalign)
    B = Guarded(p.B, dt, p.misalign)
    base = Guarded(p.base, dt, p.misalign)
    si, wi, pm = tables(p, identity=identity)
    sc = torch.from_numpy((p.scalings if scalings is None else scalings).astype(np.float32)).cuda()
    ws = lora.make_workspace(p.tok, p.nseg, p.L) if workspace else None
    lora.lora_expand(in_r.t, B.t, si, wi, pm, [int(v) for v in p.slice_offsets], sc, base.t,
                     rank=p.r, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    ok = in_r.guards_intact() and B.guards_intact() and base.guards_intact()
    return base.bits(), ok


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16).float().numpy()


def assert_close(got_bits, ref_bits, dtype, atol=2e-2, rtol=1e-2, what=""):
    """|got - ref| <= atol + rtol*|ref| elementwise; NaN/Inf must match exactly."""
    g = decode(got_bits, dtype).astype(np.float64)
    r = decode(ref_bits, dtype).astype(np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: non-finite pattern differs"
    if (~fin).any():
        assert np.array_equal(got_bits[~fin], ref_bits[~fin]), f"{what}: NaN/Inf differ"
    err = np.abs(g[fin] - r[fin])
    lim = atol + rtol * np.abs(r[fin])
    bad = err > lim
    if bad.any():
        idx = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"max err {err.max():.4g}; first {idx}: got {g[fin][idx]} "
                             f"ref {r[fin][idx]}")
    return float(err.max()) if err.size else 0.0
