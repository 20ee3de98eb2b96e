"""Helpers shared by the GPU parity tests: device transfer and the oracle-side
preparation of expected values (codes, row-major scales, tensor-core scales)."""
import numpy as np
import torch

import oracle

DEV = "cuda:0"


def dev(a, dtype=None):
    t = torch.as_tensor(a) if not isinstance(a, torch.Tensor) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


def gscale_dev(s_t) -> torch.Tensor:
    return torch.tensor([np.float32(s_t)], dtype=torch.float32, device=DEV)


def tc_to_rowmajor(tc: np.ndarray, rows: int, scols: int) -> np.ndarray:
    return oracle.scales_from_tc(tc, rows, scols)


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


# Parity bars.  Codes, scales and residues are compared bit for bit.  The GEMM
# accumulates in FP32 on the tensor cores, so its FP32 output is held to the
# relative Frobenius error 1e-4 against the binary64 oracle on the same decoded
# operands.  BF16 output adds one bf16 rounding per element (relative error at
# most 2^-9 each, 2^-8 if the FP32 result sits next to a bf16 rounding
# boundary), so it is held to 2^-8 + 1e-4 against the oracle.
GEMM_F32_TOL = 1e-4
GEMM_BF16_TOL = 2.0 ** -8 + 1e-4
