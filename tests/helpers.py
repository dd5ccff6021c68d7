"""Shared helpers of the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

import moe_inputs

POISON_BITS = 0x7FC000C7  # quiet-NaN pattern used to detect unwritten outputs
GUARD = 16                # trailing guard elements that must stay untouched
OUTPUT_REL_TOL = 1e-3     # max|y - y_ref| / max|y_ref| bar for f32 outputs
WEIGHT_REL_TOL = 1e-6     # routing weights
# The grouped FFN path multiplies the down projection in fp16 with the
# activation rounded to fp16(a * 2^-4); the oracle's act_mode 2 rounds its
# exact a the same way.  The two still differ where the kernel's f32 gate/up
# result and the exact a fall on different sides of an fp16 rounding
# midpoint (one fp16 ulp of that a), so this bar sits between the f32
# accumulation error and the output bar.
FP16_ACT_TOL = 3e-4


def bits(t: torch.Tensor) -> np.ndarray:
    return moe_inputs.bf16_bits(t)


def host(t) -> np.ndarray:
    """Host numpy copy of a tensor (numpy arrays pass through)."""
    if isinstance(t, np.ndarray):
        return t
    return t.detach().cpu().numpy()


def poisoned_f32(shape, device="cuda"):
    """f32 buffer of prod(shape) + GUARD elements filled with POISON_BITS;
    returns (full buffer, view of the logical part)."""
    n = int(np.prod(shape))
    buf = torch.full((n + GUARD,), POISON_BITS, dtype=torch.int32, device=device).view(torch.float32)
    return buf, buf[:n].view(*shape)


def assert_overwritten_and_guarded(buf: torch.Tensor, n: int):
    raw = buf.view(torch.int32).cpu().numpy()
    logical = buf[:n].cpu().numpy()
    assert not (raw[:n] == POISON_BITS).any(), "some outputs were never written"
    assert np.isfinite(logical).all(), "non-finite outputs"
    assert (raw[n:] == POISON_BITS).all(), "guard region was overwritten"


def rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max(initial=0.0) / max(np.abs(b).max(initial=0.0), 1e-300))


def sample_tokens(m: int, count: int, seed: int = 0) -> np.ndarray:
    """Seeded sorted sample of token indices, always including the first and last."""
    rng = np.random.default_rng(seed)
    picks = rng.choice(m, size=min(count, m), replace=False)
    picks = np.unique(np.concatenate([picks, [0, m - 1]]))
    return picks.astype(np.int32)
