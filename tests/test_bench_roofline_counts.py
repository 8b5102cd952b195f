"""Host-side pins of the algorithmic bytes and FLOPs that bench.py divides by
the measured kernel time (CPU only).  Each expected value is the count
written out term by term for the bench's workloads, so a dropped or doubled
term in a formula (a missing output, the state counted once, a wrong
element size) fails here."""
import os

import pytest

import bench

MB = 1 << 20


def test_layer_forward_bytes_and_flops():
    # B4 T4096 H16 dk=dv=128, bf16 q/k/v/o, fp32 log alpha and beta, fp32 S0 and S_T
    B, T, H, d = 4, 4096, 16, 128
    per_token_head = 3 * d * 2 + d * 2 + 4 + 4  # q, k, v in; o out; two fp32 gates
    states = 2 * B * H * d * d * 4             # S0 read, S_T written
    assert bench.fwd_bytes(B, T, H, d, d) == B * T * H * per_token_head + states == 278_921_216
    # per token-head: three dk x dv products (W S^T, Q S^T, the state update)
    # and, per chunk of 64, K K^T, Q K^T, W (dk) and U^g, P U (dv)
    per_flops = 3 * 2 * d * d + 2 * 64 * (3 * d + 2 * d)
    assert per_flops == 180_224
    assert bench.fwd_flops(B, T, H, d, d) == B * T * H * per_flops == 47_244_640_256


def test_decode_step_bytes():
    # B256 H16 d128: the fp32 state read and written, q, k, v in, o out (bf16),
    # log alpha and beta (fp32) per head
    B, H, d = 256, 16, 128
    expect = B * H * (2 * d * d * 4 + 4 * d * 2 + 2 * 4)
    assert bench.step_bytes(B, H, d, d) == expect == 541_097_984


def test_gdn2_bytes():
    # per token-head: q, k, v in and o out (bf16); log alpha, b (dk) and w (dv) fp32
    B, T, H, d = 4, 4096, 16, 128
    assert bench.gdr2_bytes(B, T, H, d, d) == B * T * H * (4 * d * 2 + 3 * d * 4) + 2 * B * H * d * d * 4
    assert 4 * d * 2 + 3 * d * 4 == 2560
    # decode: state read and written, q, k, v, o (bf16), three fp32 gate vectors
    assert bench.step2_bytes(256, 16, d, d) == 256 * 16 * (2 * d * d * 4 + 4 * d * 2 + 3 * d * 4)


def test_block_bytes():
    B, T, H, d, K = 4, 4096, 16, 128, 4
    taps = 3 * H * d * (K + 1) * 4  # fp32 taps and biases of the three streams
    # prologue: x in, y out for q, k, v (bf16)
    assert bench.prologue_bytes(B, T, H, d, d, K) == 2 * 3 * B * T * H * d * 2 + taps
    assert bench.prologue_bytes(B, T, H, d, d, K) == 402_653_184 + 122_880
    # prologue backward: x and dy in, dx out; taps in, their gradients out
    assert bench.prologue_bwd_bytes(B, T, H, d, d, K) == 3 * 3 * B * T * H * d * 2 + 2 * taps
    assert 9 * d * 2 == 2304
    # epilogue: o and g in, y out; backward: o, g, dy in, do and dg out
    assert bench.epilogue_bytes(B, T, H, d) == 3 * B * T * H * d * 2 + d * 4
    assert bench.epilogue_bwd_bytes(B, T, H, d) == 5 * B * T * H * d * 2 + 2 * d * 4


def test_backward_flops():
    # per token-head: 12 d^2 (six dk x dv products) + 20 C d + 4 C^2
    assert bench.bwd_flops(1, 1, 1, 128) == 12 * 128 * 128 + 20 * 64 * 128 + 4 * 64 * 64 == 376_832


def test_recorded_traffic_needs_the_recorded_source(tmp_path, monkeypatch):
    """The ncu traffic figure is reported only while the kernel source it was
    taken from is unchanged: a profile whose recorded hash does not match
    gives None."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    import hashlib
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()
    (prof / "kern.md").write_text(
        "- kernel_source: `k.cuh`\n- kernel_source_sha256: `%s`\n- traffic_bytes_per_launch: `123`\n" % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("kern") == 123
    src.write_text("kernel v2\n")
    assert bench.traffic_from_profile("kern") is None
    assert bench.traffic_from_profile("missing") is None
