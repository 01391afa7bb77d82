"""Host-side layer statistics (mxfp_block_scaled_b200/layers.py) on
hand-made results, without a GPU: SSE(chosen) / SSE(RTN) - 1 from the
verifier's per-tensor error sums, and the M=4 fraction from the per-group
counts."""
import torch

from mxfp_block_scaled_b200 import layers


def _res(err_gu, err_dn, m4_gu=None, m4_dn=None, E=2):
    def stack(err, m4, rows, cols):
        return {"sum_sq_err": torch.tensor(err, dtype=torch.float64),
                "codes": torch.zeros((E, rows, cols // 2), dtype=torch.uint8),
                "m4_count": torch.tensor(m4 if m4 is not None else [0] * E, dtype=torch.int32)}
    return {"gate_up": stack(err_gu, m4_gu, 8, 32), "down": stack(err_dn, m4_dn, 16, 16)}


def test_sse_vs_rtn():
    chosen = [_res([1.0, 2.0, 3.0, 4.0], [1.0, 1.0]), _res([0.5] * 4, [0.5, 0.5])]
    rtn = [_res([2.0, 2.0, 4.0, 4.0], [2.0, 2.0]), _res([1.0] * 4, [1.0, 1.0])]
    # (10 + 2 + 2 + 1) / (12 + 4 + 4 + 2) - 1
    assert abs(layers.sse_vs_rtn(chosen, rtn) - (15.0 / 22.0 - 1.0)) < 1e-15
    assert layers.sse_vs_rtn(rtn, rtn) == 0.0


def test_m4_fraction():
    # gate_up: 2 experts x 8 rows x 32 cols = 32 blocks; down: 2 x 16 x 16 = 32 blocks
    r = _res([0.0] * 4, [0.0] * 2, m4_gu=[3, 5], m4_dn=[0, 8])
    assert layers.m4_fraction([r]) == 16 / 64
