"""The oracle's E4M3 and E2M1 encoders against the GPU's conversion
instructions (cvt.rn.satfinite.e4m3x2.f32 / e2m1x2.f32), which the activation
kernel uses for NVFP4 block scales and elements (DiRotQ abstract: NVFP4 on
Blackwell; OCP Microscaling E4M3 / E2M1 element formats).

Inputs: every FP32 binade from well below the formats' smallest subnormal to
far above their largest value, at a fixed mantissa stride, both signs; every
representable value and every midpoint between neighbours, each with its two
FP32 neighbours; signed zeros, FP32 subnormals and the saturation edges.  The
GPU bytes must equal the oracle's bit for bit."""
import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import rq

torch = pytest.importorskip("torch")

F32 = np.float32


def _neighbours(v):
    v = np.asarray(v, F32)
    return np.concatenate([v, np.nextafter(v, F32(np.inf)), np.nextafter(v, F32(-np.inf))])


def _inputs():
    parts = []
    # binades 2^-16 .. 2^12 at a mantissa stride of 2^7 (65536 values per binade)
    mant = np.arange(0, 1 << 23, 1 << 7, dtype=np.uint32)
    for e in range(-16, 13):
        parts.append(((np.uint32(e + 127) << 23) | mant).view(F32))
    for grid in (orc.E4M3_GRID, orc.E2M1_GRID):
        g = grid.astype(F32)
        mids = ((grid[1:] + grid[:-1]) / 2).astype(F32)
        parts += [_neighbours(g), _neighbours(mids)]
    parts.append(np.array([0.0, 1e-45, 1e-40, 1.1754942e-38, 448.0, 464.0, 479.9, 480.0, 6.0, 6.5, 7.0, 1e6, 3.0e38],
                          F32))
    v = np.concatenate(parts)
    v = np.concatenate([v, -v])
    if v.size % 2:
        v = np.append(v, F32(0.0))
    return v


@pytest.mark.gpu
def test_conversions_match_the_oracle_encoders():
    v = _inputs()
    x = torch.from_numpy(v).cuda()
    e4 = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    e2 = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    rq.rq_convert_check(x, e4, e2)
    torch.cuda.synchronize()
    g4, g2 = e4.cpu().numpy(), e2.cpu().numpy()
    o4, o2 = orc.e4m3_encode(v), orc.e2m1_encode(v)
    bad4 = np.nonzero(g4 != o4)[0]
    bad2 = np.nonzero(g2 != o2)[0]
    assert bad4.size == 0, [(float(v[i]), hex(g4[i]), hex(o4[i])) for i in bad4[:8]]
    assert bad2.size == 0, [(float(v[i]), hex(g2[i]), hex(o2[i])) for i in bad2[:8]]
    assert v.size > 3_000_000
