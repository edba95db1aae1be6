"""The Python binding's marshalling, on the CPU: every wrapper is driven against a stand-in
for libw4a8 that converts each argument through the entry point's declared ctypes
signature (so a wrong argument count or type fails), with tensors of exactly the layout
size (the call goes through, each tensor's own pointer is passed) and with each sized
tensor one element short (refused before the library is reached: the kernels would
otherwise read or write past it). The device check is replaced by one that accepts CPU
tensors; with the real one, a CPU tensor is refused."""
import ctypes

import pytest
import torch

import block_quantized_w4a8_b200 as w4a8

M, N, K, G = 3, 64, 256, 64


class FakeLib:
    def __init__(self):
        self.calls = []
        for name, (res, argtypes) in w4a8.SIGNATURES.items():
            setattr(self, name, self._entry(name, res, argtypes))

    def _entry(self, name, res, argtypes):
        def call(*args):
            assert len(args) == len(argtypes), f"{name}: {len(args)} arguments, declared {len(argtypes)}"
            conv = [t.from_param(a) for t, a in zip(argtypes, args)]
            self.calls.append((name, args, conv))
            if res is ctypes.c_size_t:
                return 1 << 20
            if res is ctypes.c_char_p:
                return b""
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(w4a8, "_lib", lib)
    monkeypatch.setattr(w4a8, "_device", lambda t: t.get_device())
    monkeypatch.setattr(w4a8, "_stream", lambda s: None)
    return lib


def t(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


def cases():
    """(C entry point, wrapper, default tensor arguments, other arguments, tensors that set
    the call's dimensions and so are never cut short)."""
    i16, u8, i32, bf16 = torch.int16, torch.uint8, torch.int32, torch.bfloat16
    q40 = dict(qs=t(N, K // 2, dtype=u8), d=t(N, K // 32, dtype=i16))
    aff = dict(q=t(N, K // 8, dtype=i32), scale=t(N, K // G, dtype=i16), bias=t(N, K // G, dtype=i16))
    ws = t(4096, dtype=u8)
    x, y = t(M, K), t(M, N)
    return [
        ("w4a8_pack_q4_0", w4a8.w4a8_pack_q4_0, dict(w=t(N, K), **q40), {}, {"w"}),
        ("w4a8_quant_act_q8_0", w4a8.w4a8_quant_act_q8_0,
         dict(x=x, qx=t(M, K, dtype=torch.int8), dx=t(M, K // 32), sx=t(M, K // 32, dtype=i32)), {}, {"x"}),
        ("w4a8_gemm", w4a8.w4a8_gemm, dict(x=x, **q40, y=y, ws=ws), {}, {"x", "qs", "ws"}),
        ("w4a8_gemm_ex", w4a8.w4a8_gemm_ex, dict(x=x, **q40, y=y, ws=ws), {"path": 2}, {"x", "qs", "ws"}),
        ("w4a8_gemm_epi", w4a8.w4a8_gemm_epi, dict(x=x, **q40, y=t(M, N, dtype=bf16), ws=ws, bias=t(N)), {},
         {"x", "qs", "ws"}),
        ("w4a8_gemm_noalloc", w4a8.w4a8_gemm_noalloc, dict(x=x, **q40, y=y), {}, {"x", "qs"}),
        ("w4a8_gemm_prepared", w4a8.w4a8_gemm_prepared, dict(**q40, y=y, ws=ws), {"M": M, "K": K}, {"qs", "ws"}),
        ("w4a8_pack_affine", w4a8.w4a8_pack_affine, dict(w=t(N, K), **aff), {"group": G}, {"w"}),
        ("w4a8_gemm_affine", w4a8.w4a8_gemm_affine, dict(x=x, **aff, y=y, ws=ws), {"group": G}, {"x", "q", "ws"}),
        ("w4a8_gemm_affine_ex", w4a8.w4a8_gemm_affine_ex, dict(x=x, **aff, y=y, ws=ws), {"group": G, "path": 1},
         {"x", "q", "ws"}),
        ("w4a8_gemm_affine_epi", w4a8.w4a8_gemm_affine_epi,
         dict(x=x, q=aff["q"], scale=aff["scale"], bias_w=aff["bias"], y=t(M, N, dtype=bf16), ws=ws,
              bias=t(N, dtype=bf16)), {"group": G}, {"x", "q", "ws"}),
        ("w4a8_gemm_affine_prepared", w4a8.w4a8_gemm_affine_prepared, dict(**aff, y=y, ws=ws),
         {"M": M, "K": K, "group": G}, {"q", "ws"}),
        ("w4a8_pack_affine_nbit", w4a8.w4a8_pack_affine_nbit,
         dict(w=t(N, K), q=t(N, K * 6 // 8, dtype=u8), scale=aff["scale"], bias=aff["bias"]),
         {"group": G, "bits": 6}, {"w"}),
        ("w4a8_gemm_affine_nbit", w4a8.w4a8_gemm_affine_nbit,
         dict(x=x, q=t(N, K, dtype=u8), scale=aff["scale"], bias_w=aff["bias"], y=y, ws=ws, bias=t(N)),
         {"group": G, "bits": 8}, {"x", "q", "ws"}),
        ("w4a8_gemv_q4_k", w4a8.w4a8_gemv_q4_k, dict(x=x, w_q4k=t(N, K // 256 * 144, dtype=u8), y=y), {},
         {"x", "w_q4k"}),
        ("w4a8_gemv_q4_k_backward", w4a8.w4a8_gemv_q4_k_backward,
         dict(dy=t(M, N), w_q4k=t(N, K // 256 * 144, dtype=u8), dx=t(M, K), ws=ws), {}, {"dy", "ws"}),
        ("w4a8_prepare_act", w4a8.w4a8_prepare_act, dict(x=x, ws=ws), {}, {"x", "ws"}),
    ]


def short(v):
    """The same tensor one element short (the last axis, or the first one where the last
    axis sets a dimension of the call)."""
    if v.dim() == 1:
        return v[:-1].clone()
    return v[:, :-1].contiguous()


CASES = cases()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_exact_sizes_pass_and_marshal_the_tensors(fake, case):
    name, fn, tensors, other, _ = case
    fn(**tensors, **other)
    assert [c[0] for c in fake.calls] == [name]
    _, args, _ = fake.calls[0]
    ptrs = {a.value for a in args if isinstance(a, ctypes.c_void_p) and a.value}
    for key, v in tensors.items():
        if key == "bias" and name in ("w4a8_gemm_epi", "w4a8_gemm_affine_epi", "w4a8_gemm_affine_nbit"):
            continue  # the output bias travels inside the epilogue structure
        assert v.data_ptr() in ptrs, f"{name}: {key} not passed"


SHORT = [(c, key) for c in CASES for key, v in c[2].items() if key not in c[4]]


@pytest.mark.parametrize("case,key", SHORT, ids=[f"{c[0]}-{k}" for c, k in SHORT])
def test_a_short_tensor_is_refused_before_the_library(fake, case, key):
    name, fn, tensors, other, _ = case
    args = dict(tensors)
    if name == "w4a8_gemv_q4_k_backward" and key == "dx":
        args[key] = tensors[key][:-1].clone()  # the last axis of dx sets K
    else:
        args[key] = short(tensors[key])
    with pytest.raises(ValueError, match=rf"libw4a8: {key} holds"):
        fn(**args, **other)
    assert fake.calls == []


def test_an_output_of_the_wrong_element_size_is_refused(fake):
    """The plain entry points write f32: a bf16 y of M x N holds half the bytes."""
    tensors = CASES[2][2]
    with pytest.raises(ValueError, match="libw4a8: y holds"):
        w4a8.w4a8_gemm(tensors["x"], tensors["qs"], tensors["d"], t(M, N, dtype=torch.bfloat16), tensors["ws"])
    assert fake.calls == []


def test_host_tensors_are_refused_by_the_device_check(monkeypatch):
    monkeypatch.setattr(w4a8, "_lib", FakeLib())
    name, fn, tensors, other, _ = CASES[2]
    with pytest.raises(ValueError, match="device tensors"):
        fn(**tensors, **other)
