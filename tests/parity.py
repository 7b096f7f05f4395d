"""Helpers shared by the GPU parity tests (comparison rules and sampling)."""
import numpy as np
import torch

# fp32 outputs: within 1e-5 relative error of the oracle, and exactly zero
# where the oracle's output is zero.  (With the fixed multiply order the two
# agree bit for bit; the tolerance is the contract, not the expectation.)
Y_RTOL = 1e-5


def assert_y_close(y, y_ref, what=""):
    y = np.asarray(y, dtype=np.float32)
    y_ref = np.asarray(y_ref, dtype=np.float32)
    assert y.shape == y_ref.shape, what
    zero = y_ref == 0
    assert np.all(y[zero] == 0), f"{what}: nonzero where the oracle is zero"
    nz = ~zero
    if nz.any():
        rel = np.abs(y[nz].astype(np.float64) - y_ref[nz]) / np.abs(y_ref[nz].astype(np.float64))
        assert rel.max() <= Y_RTOL, f"{what}: max rel err {rel.max():.3e}"


def assert_acc_equal(acc, acc_ref, what=""):
    acc = np.asarray(acc)
    acc_ref = np.asarray(acc_ref)
    bad = np.argwhere(acc != acc_ref)
    assert bad.size == 0, f"{what}: {len(bad)} int32 mismatches, first at {bad[:4].tolist()}"


def sample_positions(m, n, count, seed):
    """Random (token, row) positions plus the four corners and the last row tile."""
    rng = np.random.default_rng(seed)
    pm = list(rng.integers(0, m, count))
    pn = list(rng.integers(0, n, count))
    for a, b in [(0, 0), (0, n - 1), (m - 1, 0), (m - 1, n - 1)]:
        pm.append(a)
        pn.append(b)
    tail = np.arange(max(0, n - 130), n)
    pm += list(rng.integers(0, m, len(tail)))
    pn += list(tail)
    return np.array(pm, dtype=np.int64), np.array(pn, dtype=np.int64)


def column_sum_identity(acc, xq, t):
    """sum_n acc[m,n] == sum_k xq[m,k] * (sum_n t[n,k]) for every token m.

    An exact int64 identity over the whole output, computed from the
    generator's ternary matrix; it catches a missing, repeated or misplaced
    tile anywhere at any size.
    """
    colsum = t.to(torch.int64).sum(dim=0)                 # [K]
    want = (xq.to(torch.int64) * colsum[None, :]).sum(dim=1)  # [M]
    got = acc.to(torch.int64).sum(dim=1)
    return torch.equal(got.cpu(), want.cpu())


# Guard bands: outputs the GPU tests hand to the library are views into a
# larger buffer whose bytes before and after the view hold a known pattern,
# so a write past a ragged edge into a neighbouring allocation fails a test
# even though the in-range comparison cannot see it.
GUARD_BYTES = 512
GUARD_FILL = 0xA5


def guarded_empty(shape, dtype, device="cuda"):
    """(view, buffer): a contiguous `shape` view with GUARD_BYTES of pattern on
    each side.  The view starts 512 bytes into the buffer, so it keeps the
    buffer's 256-byte alignment."""
    numel = 1
    for s in shape:
        numel *= int(s)
    esize = torch.empty((), dtype=dtype).element_size()
    g = GUARD_BYTES // esize
    buf = torch.empty(numel + 2 * g, dtype=dtype, device=device)
    buf.view(torch.uint8).fill_(GUARD_FILL)
    return buf[g:g + numel].view(*shape), buf


def guards_intact(buf) -> bool:
    """True if both guard bands of a guarded_empty buffer still hold the pattern."""
    b = buf.view(torch.uint8).cpu()
    return bool((b[:GUARD_BYTES] == GUARD_FILL).all() and (b[-GUARD_BYTES:] == GUARD_FILL).all())
