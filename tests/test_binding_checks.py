"""The Python binding rejects, on the host, arguments whose sizes the C ABI
cannot see: a buffer of the wrong type or shape, a tensor on another device.

Each case must raise EPError before any CUDA call, so a handle object is
built without a device workspace (its attributes set by hand) and the
tensors are CPU tensors.  Against a handle "on" cuda:0 every CPU tensor must
be refused; against a handle "on" the CPU, the dtype and shape checks that
come after the device check are reached and must refuse the bad buffer.
"""
import ctypes

import pytest
import torch


@pytest.fixture(scope="module")
def ep():
    import combine_ep_layout_08_b200 as mod
    from combine_ep_layout_08_b200 import _build

    _build.build()
    mod.load_library()
    return mod


T, K, E, R, H = 16, 4, 8, 2, 256


def fake_handle(ep, device):
    h = object.__new__(ep.EPHandle)
    h.device = torch.device(device)
    h.max_tokens, h.k, h.E, h.R, h.block_m = T, K, E, R, 128
    h.T = T
    h._h = ctypes.c_void_p()
    return h


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def fp8(*shape):
    return torch.zeros(shape, dtype=torch.float8_e4m3fn)


def refused(fn, *args, why=None):
    """fn(*args) raises EPError(EP_ERR_INVALID_ARG) whose message holds `why`."""
    with pytest.raises(Exception) as info:
        fn(*args)
    assert type(info.value).__name__ == "EPError", repr(info.value)
    assert info.value.status == 1  # EP_ERR_INVALID_ARG
    if why is not None:
        assert why in str(info.value), str(info.value)


def test_host_tensors_are_refused_by_a_device_handle(ep):
    h = fake_handle(ep, "cuda:0")
    idx = torch.zeros((T, K), dtype=torch.int64)
    on = "must be on cuda:0"
    refused(ep.ep_layout, h, idx, why=on)
    refused(ep.ep_layout_dispatch, h, idx, bf16(T, H), "bf16", bf16(64, H), why=on)
    refused(ep.ep_dispatch, h, bf16(T, H), "bf16", bf16(64, H), why=on)
    refused(ep.ep_combine, h, bf16(64, H), f32(T, K), bf16(T, H), why=on)
    refused(ep.ep_dispatch_range, h, 0, bf16(4, H), "bf16", bf16(64, H), why=on)
    refused(ep.ep_combine_range, h, 0, bf16(64, H), f32(4, K), bf16(4, H), why=on)
    refused(ep.ep_dispatch_backward, h, bf16(64, H), bf16(T, H), why=on)
    refused(ep.ep_combine_backward, h, bf16(T, H), bf16(64, H), f32(T, K), bf16(64, H), why=on)
    refused(ep.ep_dispatch_weights, h, f32(T, K), f32(64), why=on)
    refused(ep.ep_zero_pad_rows, h, bf16(64, H), why=on)
    refused(ep.ep_dispatch_ranks, h, 0, bf16(4, H), "bf16", [bf16(32, H)] * R, why=on)
    # per-rank buffers may be other GPUs' (peers) but must be CUDA tensors
    rank = "per-rank buffers must be 2-D cuda"
    refused(ep.ep_combine_ranks, h, 0, [bf16(32, H)] * R, f32(4, K), bf16(4, H), why=rank)
    refused(ep.ep_dispatch_ranks_backward, h, 0, [bf16(32, H)] * R, bf16(4, H), why=rank)
    refused(ep.ep_combine_ranks_backward, h, 0, bf16(4, H), [bf16(32, H)] * R, f32(4, K),
            [bf16(32, H)] * R, why=rank)


def test_range_receive_buffer_must_match_the_format(ep):
    h = fake_handle(ep, "cpu")
    x = bf16(4, H)
    rx, no_sc = "recv_x must be contiguous", "FP8 needs contiguous f32 recv_scales"
    refused(ep.ep_dispatch_range, h, 0, x, "bf16", fp8(64, H), why=rx)     # 1-byte rows, a copy
    refused(ep.ep_dispatch_range, h, 0, x, "fp8", bf16(64, H), why=rx)     # 2-byte rows for FP8
    refused(ep.ep_dispatch_range, h, 0, x, "bf16", bf16(64, H + 8), why=rx)
    refused(ep.ep_dispatch_range, h, 0, x, "fp8", fp8(64, H), why=no_sc)
    refused(ep.ep_dispatch_range, h, 0, x, "fp8", fp8(64, H),
            torch.zeros((64, H // 128), dtype=torch.float64), why=no_sc)
    rm, mn = "recv_scales must be f32 [cap, H/128]", "recv_scales must be f32 [H/128, cap]"
    refused(ep.ep_dispatch_range, h, 0, x, "fp8", fp8(64, H), f32(63, H // 128), why=rm)
    refused(ep.ep_dispatch_range, h, 0, x, "fp8", fp8(64, H), f32(64, H // 64), why=rm)
    refused(ep.ep_dispatch_range, h, 0, x, "fp8_mn", fp8(64, H), f32(64, H // 128), why=mn)


def test_dispatch_receive_buffers_are_checked(ep):
    h = fake_handle(ep, "cpu")
    x = bf16(T, H)
    refused(ep.ep_dispatch, h, x, "bf16", fp8(64, H), why="recv_x must be contiguous")
    refused(ep.ep_dispatch, h, x, "fp8", fp8(64, H), f32(10, H // 128),
            why="recv_scales must be f32 [cap, H/128]")
    refused(ep.ep_dispatch, h, x, "fp8_mn", fp8(64, H), f32(H // 128, 60),
            why="recv_scales must be f32 [H/128, cap]")
    refused(ep.ep_dispatch, h, bf16(T - 1, H), "bf16", bf16(64, H),   # not the layout's T
            why="x must be contiguous bf16/fp16 [T, H]")


def test_backward_and_weights_shapes_are_checked(ep):
    h = fake_handle(ep, "cpu")
    y = bf16(64, H)
    go = "grad_out must be [T, H]"
    refused(ep.ep_combine_backward, h, bf16(T - 1, H), y, f32(T, K), bf16(64, H), why=go)
    refused(ep.ep_combine_backward, h, bf16(T, H + 8), y, f32(T, K), bf16(64, H), why=go)
    refused(ep.ep_combine_backward, h, bf16(T, H), y, f32(T, K), bf16(64, H + 8),
            why="grad_y must be [*, H]")
    refused(ep.ep_dispatch_backward, h, y, bf16(T - 1, H), why="grad_x must be [T, H]")
    rw = "recv_weights must be f32 [cap]"
    refused(ep.ep_dispatch_weights, h, f32(T, K), bf16(64), why=rw)       # 2-byte weights
    refused(ep.ep_dispatch_weights, h, f32(T, K), f32(64, 1), why=rw)     # not 1-D
    refused(ep.ep_dispatch_weights, h, f32(T, K + 1), f32(64), why="topk_weights must be f32 [T, k]")
    refused(ep.ep_combine_range, h, 0, y, f32(4, K), bf16(4 * H), why="must be 2-D")


def test_rank_buffers_are_checked(ep):
    h = fake_handle(ep, "cpu")
    x = bf16(4, H)
    ok = [bf16(32, H) for _ in range(R)]
    one = "one buffer per rank"
    refused(ep.ep_dispatch_ranks, h, 0, x, "bf16", ok[:1], why=one)
    refused(ep.ep_dispatch_ranks, h, 0, x, "fp8", [fp8(32, H)] * R, why=one)   # no scales
    refused(ep.ep_dispatch_ranks, h, 0, x, "bf16", [bf16(32, H), fp8(32, H)],
            why="recv_x must be contiguous")
    refused(ep.ep_dispatch_ranks, h, 0, x, "fp8", [fp8(32, H)] * R,
            [f32(32, H // 128), f32(31, H // 128)],                        # rank 1's scales short
            why="recv_scales must be f32 [cap, H/128]")
    refused(ep.ep_combine_ranks, h, 0, [bf16(32, H), bf16(32 * H)], f32(4, K), bf16(4, H),
            why="per-rank buffers must be 2-D")
    refused(ep.ep_combine_ranks, h, 0, ok, f32(4, K), bf16(4 * H), why="out_rows must be 2-D")
    refused(ep.ep_dispatch_ranks_backward, h, 0, ok, bf16(4 * H), why="grad_x_rows must be 2-D")
    refused(ep.ep_combine_ranks_backward, h, 0, bf16(4 * H), ok, f32(4, K), ok,
            why="grad_out_rows must be 2-D")


class Reached(Exception):
    """Raised where the binding would make the device current and call the library."""


def test_valid_arguments_pass_every_check(ep, monkeypatch):
    def stop(h):
        raise Reached()

    monkeypatch.setattr(ep, "_on", stop)
    h = fake_handle(ep, "cpu")
    idx = torch.zeros((T, K), dtype=torch.int64)
    x, y, w = bf16(T, H), bf16(64, H), f32(T, K)
    rank = [bf16(32, H) for _ in range(R)]
    calls = [
        (ep.ep_layout, h, idx),
        (ep.ep_layout_dispatch, h, idx, x, "fp8"),
        (ep.ep_layout_dispatch, h, idx, x.half(), None),
        (ep.ep_dispatch, h, x),
        (ep.ep_dispatch, h, x, "fp8"),
        (ep.ep_dispatch, h, x, "fp8_mn"),
        (ep.ep_dispatch, h, x.half(), "fp8"),
        (ep.ep_dispatch, h, x, "fp8", fp8(64, H), f32(80, H // 128)),   # more scale rows than cap
        (ep.ep_combine, h, y, w),
        (ep.ep_combine, h, y.half(), w),
        (ep.ep_dispatch_range, h, 0, x[:4], "bf16", y),
        (ep.ep_dispatch_range, h, 4, x[4:4], "fp8", fp8(64, H), f32(64, H // 128)),
        (ep.ep_dispatch_range, h, 0, x[:4], "fp8_mn", fp8(64, H), f32(H // 128, 64)),
        (ep.ep_combine_range, h, 0, y, w[:4], bf16(4, H)),
        (ep.ep_dispatch_backward, h, y),
        (ep.ep_combine_backward, h, x, y, w),
        (ep.ep_combine_backward, h, x.half(), y.half(), w, bf16(70, H).half()),
        (ep.ep_dispatch_weights, h, w),
        (ep.ep_dispatch_weights, h, w, f32(64)),
        (ep.ep_zero_pad_rows, h, f32(64, 3)),
        (ep.ep_dispatch_ranks, h, 0, x[:4], "bf16", rank),
        (ep.ep_dispatch_ranks, h, 0, x[:4], "fp8", [fp8(32, H), fp8(0, H)],
         [f32(32, H // 128), f32(0, H // 128)]),
        (ep.ep_combine_ranks, h, 0, rank, w[:4], bf16(4, H)),
        (ep.ep_dispatch_ranks_backward, h, 0, rank, bf16(4, H)),
        (ep.ep_combine_ranks_backward, h, 0, bf16(4, H), rank, w[:4], rank),
    ]
    for fn, *args in calls:
        with pytest.raises(Reached):
            fn(*args)
