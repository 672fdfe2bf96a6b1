"""Shared helpers for the GPU parity tests: moving tensors, comparing the CUDA
path's outputs with the oracle's, and Freivalds' check of an int32 product."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from w8a8_post_quantization_calibrate_b200 import synth


def host(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> numpy (bf16 as uint16 bits)."""
    return synth.host_array(t.detach().cpu())


def bits32(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_bitexact_f32(got: np.ndarray, want: np.ndarray, what: str) -> None:
    g, w = bits32(got), bits32(want)
    if not np.array_equal(g, w):
        idx = np.argwhere(g != w)
        i = tuple(idx[0])
        raise AssertionError(f"{what}: {len(idx)} mismatches, first at {i}: got {got[i]!r} want {want[i]!r}")


def assert_equal(got: np.ndarray, want: np.ndarray, what: str) -> None:
    if not np.array_equal(got, want):
        idx = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(idx)} mismatches, first at {idx[:3].tolist()}: "
                             f"got {got[tuple(idx[0])]} want {want[tuple(idx[0])]}")


def assert_f32_close(got: np.ndarray, want: np.ndarray, what: str, rtol: float = 1e-6) -> int:
    """|got - want| <= rtol * |want| elementwise (fp32 output tolerance).
    Returns the number of bit-exact elements."""
    g = got.astype(np.float64)
    w = want.astype(np.float64)
    err = np.abs(g - w)
    lim = rtol * np.abs(w)
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{what}: {len(bad)} outside {rtol} rel, first {bad[:3].tolist()}"
    return int(np.sum(bits32(got) == bits32(want)))


def assert_bf16_within_ulp(got_bits: np.ndarray, want_bits: np.ndarray, what: str, ulps: int = 1) -> int:
    """bf16 outputs (uint16 bit patterns) within `ulps` units in the last place.
    Returns the number of bit-exact elements."""
    g = got_bits.astype(np.int32)
    w = want_bits.astype(np.int32)
    # map sign-magnitude bit patterns onto a monotone integer line
    g = np.where(g & 0x8000, -(g & 0x7FFF), g)
    w = np.where(w & 0x8000, -(w & 0x7FFF), w)
    d = np.abs(g - w)
    assert d.max(initial=0) <= ulps, f"{what}: max {d.max()} bf16 ulps apart at {np.argwhere(d > ulps)[:3].tolist()}"
    return int(np.sum(got_bits == want_bits))


def freivalds(acc: np.ndarray, xq: np.ndarray, wq: np.ndarray, rounds: int = 3, seed: int = 0,
              chunk: int = 1024) -> None:
    """Freivalds' randomized check (1977) that acc == xq @ wq^T exactly:
    acc r == xq (wq^T r) for random r in {-3..3}^N, O(MN + NK + MK) work.

    Evaluated with float BLAS in row chunks, which is exact here: every partial
    sum is an integer, below 2^24 for the float32 products wq^T r
    (127 * 3 * chunk) and below 2^53 for the float64 ones (127^2 K * 3 N)."""
    rng = np.random.default_rng(seed)
    M, N = acc.shape
    K = xq.shape[1]
    assert 127 * 127 * K * 3 * N < 2 ** 53 and 127 * 3 * chunk < 2 ** 24
    for _ in range(rounds):
        r = rng.integers(-3, 4, size=N)
        wr = np.zeros(K, np.float64)
        for i in range(0, N, chunk):
            wr += (r[i:i + chunk].astype(np.float32) @ wq[i:i + chunk].astype(np.float32)).astype(np.float64)
        rf = r.astype(np.float64)
        for i in range(0, M, chunk):
            lhs = acc[i:i + chunk].astype(np.float64) @ rf
            rhs = xq[i:i + chunk].astype(np.float64) @ wr
            bad = np.nonzero(lhs != rhs)[0]
            assert bad.size == 0, f"Freivalds check failed on rows {(bad[:5] + i).tolist()}"


def oracle_rows(xq: np.ndarray, wq: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Oracle int32 accumulators for a subset of rows."""
    return oracle.gemm_i8(np.ascontiguousarray(xq[rows]), wq)


class Guarded:
    """A device output buffer with guard bands: `band` bytes of a seeded
    pattern before and after the buffer proper, which every call writing the
    buffer must leave as they were (a check for stray writes, in place of a
    memory checker). `t` is the typed view the call writes; its start is
    256-byte aligned."""

    def __init__(self, shape, dtype, device, band=4096, seed=0):
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        self.band = band
        self.nbytes = nbytes
        g = torch.Generator().manual_seed(seed)
        self.pattern = torch.randint(0, 256, (2 * band,), generator=g, dtype=torch.uint8)
        tail_pad = (-nbytes) % 256
        self.raw = torch.empty(band + nbytes + tail_pad + band, dtype=torch.uint8, device=device)
        self.raw.fill_(0x5A)
        self.raw[:band] = self.pattern[:band].to(device)
        self.raw[band + nbytes:band + nbytes + band] = self.pattern[band:].to(device)
        self.t = self.raw[band:band + nbytes].view(dtype).view(shape)

    def check(self, what: str) -> None:
        torch.cuda.synchronize()
        raw = self.raw.cpu()
        before = raw[:self.band]
        after = raw[self.band + self.nbytes:self.band + self.nbytes + self.band]
        for name, got, want in (("before", before, self.pattern[:self.band]),
                                ("after", after, self.pattern[self.band:])):
            bad = torch.nonzero(got != want).flatten()
            assert bad.numel() == 0, f"{what}: {bad.numel()} guard bytes changed {name} the buffer, first at {bad[:4].tolist()}"
