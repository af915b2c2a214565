"""Shared helpers of the parity tests (no method arithmetic here)."""
import numpy as np
import torch

# Tolerances of the layer: rel-L2 against the fp64 oracle
TOL_BF16 = 2e-3      # bf16 outputs (o, y)
TOL_STATE = 1e-4     # fp32 final recurrent state


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def dev_f32(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def dev_i32(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32).astype(np.float64)


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def ulp_diff_bf16(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of finite bf16 bit patterns."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), x + 0x8000)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def restrict_decode_heads(dec, heads):
    """The decode inputs of the value heads `heads` alone, as a layer with hk = hv = len(heads).

    Value head h reads the q and k channels of key head h // (hv / hk), its own v channels, a,
    b, A_log, dt_bias and state; nothing else enters its recurrence, so the oracle run on the
    restriction gives exactly its results on those heads (indexing only).
    """
    import gdr_inputs as GI
    d = dec.dk
    khs = [h // (dec.hv // dec.hk) for h in heads]
    chans = np.concatenate([np.arange(kh * d, (kh + 1) * d) for kh in khs]
                           + [dec.hk * d + np.arange(kh * d, (kh + 1) * d) for kh in khs]
                           + [2 * dec.hk * d + np.arange(h * d, (h + 1) * d) for h in heads])
    return GI.DecodeInputs(np.ascontiguousarray(dec.x[:, :, chans]), np.ascontiguousarray(dec.a[:, :, heads]),
                           np.ascontiguousarray(dec.b[:, :, heads]), np.ascontiguousarray(dec.conv_w[chans]),
                           np.ascontiguousarray(dec.conv_state[:, :, chans]),
                           np.ascontiguousarray(dec.state[:, heads]), dec.A_log[heads].copy(),
                           dec.dt_bias[heads].copy(), len(heads), len(heads), dec.dk, dec.dv, dec.scale)
