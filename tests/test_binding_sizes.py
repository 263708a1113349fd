"""The Python binding checks, before calling the library, that every tensor
holds the bytes the problem needs: a short buffer raises MoeError
(MOE_ERR_INVALID_ARG) instead of reaching the GPU as an out-of-bounds access.

Runs on the CPU with tensors on torch's `meta` device (sizes, no storage):
with every buffer exactly large enough the checks pass and the call stops at
the binding's "expected a CUDA tensor" check, before the library is called;
with any one buffer one element short it raises MoeError first."""
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200 import build

N, H, E, K, S = 37, 256, 16, 3, 4
ROWS = N * K + 9


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    B.load()


def m(*shape, dtype=torch.int32):
    return torch.empty(shape, dtype=dtype, device="meta")


def bf16(*shape):
    return m(*shape, dtype=torch.bfloat16)


def u8(*shape):
    return m(*shape, dtype=torch.uint8)


def f32(*shape):
    return m(*shape, dtype=torch.float32)


def problem(**kw):
    p = dict(num_tokens=N, hidden=H, num_experts=E, top_k=K, num_segments=S,
             recv_capacity=ROWS)
    p.update(kw)
    return B.Problem(**p)


def _layout_args(prob):
    ws = B.moe_workspace_bytes(prob)
    return [m(N, K), m(E), m(E + 1), m(4, S), m(prob.recv_capacity or E * prob.expert_capacity),
            m(N, K), u8(N, K), m(1), u8(ws)]


I = 96


def cases():
    """entry point name -> (problem, positional tensor arguments, leading
    non-tensor arguments)."""
    p = problem()
    sw = problem(flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES)
    cap = problem(expert_capacity=5, recv_capacity=0)
    R = ROWS
    return {
        "moe_dispatch_layout": (p, _layout_args(p), ()),
        "moe_dispatch_layout[capacity]": (cap, _layout_args(cap), ()),
        "moe_dispatch_layout_noalloc": (p, _layout_args(p)[:-1], ()),
        "moe_permute": (p, [bf16(N, H), m(R), m(N, K), bf16(R, H)], ()),
        "moe_permute_premultiplied": (p, [bf16(N, H), m(R), m(N, K), f32(N, K), bf16(R, H)], ()),
        "moe_permute_to_peers": (p, [bf16(N, H), m(R), m(N, K), m(4, S),
                                     m(S, dtype=torch.int64), m(S, dtype=torch.int64)], ()),
        "moe_permute_quant_fp8_to_peers": (p, [bf16(N, H), m(R), m(N, K), m(4, S),
                                               m(S, dtype=torch.int64), m(S, dtype=torch.int64),
                                               m(S, dtype=torch.int64)], ()),
        "moe_permute_quant_nvfp4_to_peers": (p, [bf16(N, H), m(R), m(N, K), m(4, S), f32(1),
                                                 m(S, dtype=torch.int64),
                                                 m(S, dtype=torch.int64),
                                                 m(S, dtype=torch.int64)], ()),
        "moe_permute_quant_fp8": (p, [bf16(N, H), m(R), m(N, K), u8(R, H), f32(R, H // 128)], ()),
        "moe_permute_quant_nvfp4": (p, [bf16(N, H), m(R), m(N, K), f32(1), u8(R, H // 2),
                                        u8(R, H // 16)], ()),
        "moe_permute_quant_nvfp4[atoms]": (sw, [bf16(N, H), m(R), m(N, K), f32(1), u8(R, H // 2),
                                               u8(B.nvfp4_swizzled_scale_bytes(R, H))], ()),
        "moe_permute_quant_mxfp4": (p, [bf16(N, H), m(R), m(N, K), u8(R, H // 2),
                                        u8(R, H // 32)], ()),
        "moe_permute_quant_mxfp4[atoms]": (sw, [bf16(N, H), m(R), m(N, K), u8(R, H // 2),
                                               u8(B.nvfp4_swizzled_scale_bytes(R, H, 32))], ()),
        "moe_combine": (p, [bf16(R, H), f32(N, K), m(N, K), bf16(N, H)], ()),
        "moe_combine_from_peers": (p, [m(S, dtype=torch.int64), m(S, dtype=torch.int64),
                                       m(4, S), f32(N, K), m(N, K), bf16(N, H)], ()),
        "moe_permute_backward": (p, [bf16(R, H), m(N, K), bf16(N, H)], ()),
        "moe_combine_backward": (p, [bf16(N, H), bf16(R, H), f32(N, K), m(N, K), m(R),
                                     bf16(R, H), f32(N, K)], ()),
        "moe_swiglu_quant[nvfp4]": (p, [bf16(R, 2 * I), m(R), f32(1), u8(R, I // 2),
                                        u8(R, I // 16)], (I, B.MOE_QUANT_NVFP4, 0)),
        "moe_swiglu_quant[mxfp8]": (p, [bf16(R, 2 * I), m(R), None, u8(R, I), u8(R, I // 32)],
                                    (I, B.MOE_QUANT_MXFP8, 1)),
        "moe_swiglu_quant[mxfp6]": (p, [bf16(R, 2 * I), m(R), None, u8(R, 3 * I // 4),
                                        u8(R, I // 32)], (I, B.MOE_QUANT_MXFP6_E2M3, 0)),
        "moe_swiglu_quant[bf16]": (p, [bf16(R, 2 * I), m(R), None, bf16(R, I), None],
                                   (I, B.MOE_QUANT_BF16, 0)),
    }


def _call(name, prob, lead, args):
    fn = getattr(B, name.split("[")[0])
    return fn(prob, *lead, *args)


def _shrink(t):
    flat = t.reshape(-1)
    return flat[:flat.numel() - 1]


@pytest.mark.parametrize("name", sorted(cases()))
def test_exact_sizes_pass_the_size_checks(name):
    prob, args, lead = cases()[name]
    with pytest.raises(ValueError, match="CUDA tensor"):
        _call(name, prob, lead, args)


@pytest.mark.parametrize("name", sorted(cases()))
def test_every_short_buffer_raises_before_the_call(name):
    prob, args, lead = cases()[name]
    checked = 0
    for i, t in enumerate(args):
        if t is None or t.numel() == 0:
            continue
        short = list(args)
        short[i] = _shrink(t)
        with pytest.raises(B.MoeError) as e:
            _call(name, prob, lead, short)
        assert e.value.code == B.MOE_ERR_INVALID_ARG
        assert "bytes" in str(e.value)
        checked += 1
    assert checked == sum(t is not None and t.numel() > 0 for t in args)


def test_drop_mask_may_be_omitted():
    prob, args, lead = cases()["moe_dispatch_layout"]
    args = list(args)
    args[6] = None
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.moe_dispatch_layout(prob, *args)
