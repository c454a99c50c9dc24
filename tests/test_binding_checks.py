"""The Python binding checks every tensor before it calls the library: the C
ABI sees only pointers and sizes, so a tensor of the wrong type, size,
layout or device would otherwise reach a kernel that writes past its end.
The CPU cases hand the bindings host tensors (rejected before any library
call; without the checks the call would reach the library and fail there
with a CUDA status instead).  The GPU cases hand them device tensors of the
wrong size or type."""
import pytest
import torch

from exact_tiled_attention_39_b200 import attn as A


def _host(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("entry", ["mxfp8", "nvfp4", "rotated"])
def test_quantisers_reject_host_tensors(entry):
    x = _host((4, 2, 64), torch.bfloat16)
    codes = _host((4, 2, 64), torch.uint8)
    scales = _host((4, 2, 4), torch.uint8)
    with pytest.raises(ValueError):
        if entry == "mxfp8":
            A.attn_quantize_mxfp8(x, codes, scales)
        elif entry == "nvfp4":
            A.attn_quantize_nvfp4(x, codes[..., :32], scales)
        else:
            A.attn_quantize_mxfp8_rotated(x, _host((64,), torch.float32), codes, scales[..., :2])


@pytest.mark.parametrize("entry", ["fwd", "incoherent", "noalloc", "bwd"])
def test_attention_entries_reject_host_tensors(entry):
    T, H, d = 16, 2, 64
    q = _host((T, H, d), torch.bfloat16)
    lse = _host((H, T), torch.float32)
    with pytest.raises(ValueError):
        if entry == "fwd":
            A.attn_fwd(q, q, q, None, q, lse, True, 0.125)
        elif entry == "incoherent":
            A.attn_fwd_incoherent(q, q, q, None, q, lse, True, 0.125, _host((d,), torch.float32))
        elif entry == "noalloc":
            A.attn_fwd_noalloc(q, q, q, None, q, lse, True, 0.125)
        else:
            A.attn_bwd(q, q, q, q, q, lse, None, q, q, q, True, 0.125)


def test_device_error_read_rejects_host_workspace():
    with pytest.raises(ValueError):
        A.attn_get_device_error(_host((256,), torch.uint8))


# ------------------------------------------------------------------ GPU


@pytest.mark.gpu
@pytest.mark.parametrize("bad", ["codes_short", "scales_short", "codes_dtype", "x_fp32",
                                 "x_noncontig"])
@pytest.mark.parametrize("entry", ["mxfp8", "nvfp4"])
def test_quantisers_reject_bad_device_tensors(entry, bad, cuda_device):
    rows, cols = 8, 128
    code_bytes = cols if entry == "mxfp8" else cols // 2
    scale_bytes = cols // 32 if entry == "mxfp8" else cols // 16
    x = torch.zeros((rows, cols), dtype=torch.bfloat16, device=cuda_device)
    codes = torch.zeros((rows, code_bytes), dtype=torch.uint8, device=cuda_device)
    scales = torch.zeros((rows, scale_bytes), dtype=torch.uint8, device=cuda_device)
    if bad == "codes_short":
        codes = codes[:-1]
    elif bad == "scales_short":
        scales = scales[:-1]
    elif bad == "codes_dtype":
        codes = torch.zeros((rows, code_bytes // 2), dtype=torch.int16, device=cuda_device)
    elif bad == "x_fp32":
        x = x.float()
    else:
        x = torch.zeros((cols, rows), dtype=torch.bfloat16, device=cuda_device).t()
    fn = A.attn_quantize_mxfp8 if entry == "mxfp8" else A.attn_quantize_nvfp4
    with pytest.raises(ValueError):
        fn(x, codes, scales)


@pytest.mark.gpu
@pytest.mark.parametrize("bad", ["signs_len", "signs_dtype", "scales_short"])
def test_rotated_quantiser_rejects_bad_device_tensors(bad, cuda_device):
    rows, cols = 8, 128
    x = torch.zeros((rows, cols), dtype=torch.bfloat16, device=cuda_device)
    signs = torch.ones(cols, dtype=torch.float32, device=cuda_device)
    codes = torch.zeros((rows, cols), dtype=torch.uint8, device=cuda_device)
    scales = torch.zeros((rows, cols // 32), dtype=torch.uint8, device=cuda_device)
    if bad == "signs_len":
        signs = signs[:64]
    elif bad == "signs_dtype":
        signs = signs.bfloat16()
    else:
        scales = scales[:, :2]
    with pytest.raises(ValueError):
        A.attn_quantize_mxfp8_rotated(x, signs, codes, scales)
