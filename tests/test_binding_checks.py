"""The binding checks every operand's shape and dtype before a pointer reaches the library.

The C ABI takes sizes from a few arguments (x and W, the logits); a smaller
buffer passed for any other operand would be read or written past its end on
the GPU. These checks run before any device work, so they are tested here on
CPU tensors: a mismatch raises, and well-formed CPU tensors get as far as the
device check.
"""
import pytest

torch = pytest.importorskip("torch")

import sampling_gated_lora_b200 as U
import workloads as W

bf16, f32, i32, u8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def _linear(M=4, K=64, N=32, r=8, dt=bf16):
    return dict(x=torch.zeros(M, K, dtype=dt), W=torch.zeros(N, K, dtype=dt),
                A=torch.zeros(r, K, dtype=dt), Bl=torch.zeros(N, r, dtype=dt),
                gate=torch.zeros(M, dtype=u8))


def _call_linear(a, **kw):
    return U.gated_lora_linear(a["x"], a["W"], a["A"], a["Bl"], a["gate"], 1.0, **kw)


def test_well_formed_linear_reaches_the_device_check():
    with pytest.raises(ValueError, match="CUDA device"):
        _call_linear(_linear())


@pytest.mark.parametrize("name,bad,err,msg", [
    ("W", torch.zeros(32, 48, dtype=bf16), ValueError, "W has shape"),
    ("A", torch.zeros(8, 48, dtype=bf16), ValueError, "A has shape"),
    ("Bl", torch.zeros(16, 8, dtype=bf16), ValueError, "Bl has shape"),
    ("Bl", torch.zeros(32, 4, dtype=bf16), ValueError, "Bl has shape"),
    ("gate", torch.zeros(3, dtype=u8), ValueError, "gate has shape"),
    ("gate", torch.zeros(4, dtype=torch.bool), TypeError, "gate has dtype"),
    ("W", torch.zeros(32, 64, dtype=f32), TypeError, "W has dtype"),
    ("A", torch.zeros(8, 64, dtype=f32), TypeError, "A has dtype"),
])
def test_linear_operand_mismatch_raises(name, bad, err, msg):
    a = _linear()
    a[name] = bad
    with pytest.raises(err, match=msg):
        _call_linear(a)


def test_linear_output_and_missing_adapter_checks():
    a = _linear()
    with pytest.raises(ValueError, match="y has shape"):
        _call_linear(a, y=torch.zeros(4, 16, dtype=bf16))
    a["gate"] = None
    with pytest.raises(ValueError, match="gate is required"):
        _call_linear(a)
    with pytest.raises(TypeError, match="x has dtype"):
        U.gated_lora_linear(torch.zeros(4, 64, dtype=torch.float16), a["W"], a["A"], a["Bl"],
                            torch.zeros(4, dtype=u8))


def test_group_checks():
    x = torch.zeros(4, 64, dtype=bf16)
    Ws = [torch.zeros(32, 64, dtype=bf16), torch.zeros(16, 64, dtype=bf16)]
    As = [torch.zeros(8, 64, dtype=bf16)] * 2
    Bls = [torch.zeros(32, 8, dtype=bf16), torch.zeros(16, 8, dtype=bf16)]
    g = torch.zeros(4, dtype=u8)
    with pytest.raises(ValueError, match="CUDA device"):
        U.gated_lora_linear_group(x, Ws, As, Bls, g)
    with pytest.raises(ValueError, match=r"Bls\[1\] has shape"):
        U.gated_lora_linear_group(x, Ws, As, [Bls[0], Bls[0]], g)
    with pytest.raises(ValueError, match="one entry per linear"):
        U.gated_lora_linear_group(x, Ws, As[:1], Bls, g)
    with pytest.raises(ValueError, match="1 to 3 linears"):
        U.gated_lora_linear_group(x, Ws * 2, As * 2, Bls * 2, g)
    with pytest.raises(ValueError, match="ys needs 1 outputs"):
        U.gated_lora_linear_group(x, Ws, As, Bls, g, silu_pair=True,
                                  ys=[torch.zeros(4, 32, dtype=bf16)] * 2)
    with pytest.raises(ValueError, match=r"ys\[0\] has shape"):
        U.gated_lora_linear_group(x, Ws, As, Bls, g, ys=[torch.zeros(4, 16, dtype=bf16),
                                                        torch.zeros(4, 16, dtype=bf16)])


def _verify_args(B=2, k=4, V=64, dt=bf16):
    return (torch.zeros(B, k + 1, V, dtype=dt), torch.zeros(B, k, V, dtype=dt),
            torch.zeros(B, k, dtype=i32))


def test_verify_checks():
    P, Q, D = _verify_args()
    with pytest.raises(ValueError, match="CUDA device"):
        U.psi_verify(P, Q, D, 1.0, 0, 0)
    with pytest.raises(ValueError, match="q_logits has shape"):
        U.psi_verify(P, torch.zeros(2, 4, 32, dtype=bf16), D, 1.0, 0, 0)
    with pytest.raises(TypeError, match="q_logits has dtype"):
        U.psi_verify(P, Q.float(), D, 1.0, 0, 0)
    with pytest.raises(ValueError, match="draft has shape"):
        U.psi_verify(P, Q, torch.zeros(2, 3, dtype=i32), 1.0, 0, 0)
    with pytest.raises(TypeError, match="draft has dtype"):
        U.psi_verify(P, Q, D.long(), 1.0, 0, 0)
    with pytest.raises(ValueError, match="out_tokens has shape"):
        U.psi_verify(P, Q, D, 1.0, 0, 0, out_tokens=torch.zeros(2, 4, dtype=i32))
    with pytest.raises(ValueError, match="dev_status has shape"):
        U.psi_verify_noalloc(P, Q, D, 1.0, 0, 0, dev_status=torch.zeros(2, dtype=i32))
    with pytest.raises(ValueError, match="draft has shape"):
        U.draft_sample(Q, 1.0, 0, 0, draft=torch.zeros(2, 5, dtype=i32))


def test_glue_checks():
    x = torch.zeros(4, 64, dtype=bf16)
    with pytest.raises(TypeError, match="x has dtype"):
        U.rmsnorm(x.float())
    with pytest.raises(ValueError, match="y has shape"):
        U.rmsnorm(x, y=torch.zeros(4, 32, dtype=bf16))
    with pytest.raises(ValueError, match="b has shape"):
        U.silu_mul(x, torch.zeros(4, 32, dtype=bf16))


def _tiny_model_parts():
    s = W.TINY_SHAPE
    layers, head = W.model_weights_torch(s, "cpu", seed=0)
    return s, layers, head


def test_model_weights_of_the_workload_pass_the_checks():
    s, layers, head = _tiny_model_parts()
    with pytest.raises(ValueError, match="CUDA device"):
        U.Model(layers, head, s.hidden, s.q_out, s.kv_out, s.inter, s.vocab, s.r)


def test_model_weight_mismatch_raises():
    s, layers, head = _tiny_model_parts()
    Wo, Ao, Blo = layers[1]["o"]
    layers[1]["o"] = (Wo, Ao, Blo[:-8])
    with pytest.raises(ValueError, match="layer 1 o Bl has shape"):
        U.Model(layers, head, s.hidden, s.q_out, s.kv_out, s.inter, s.vocab, s.r)
    layers[1]["o"] = (Wo, Ao, Blo)
    with pytest.raises(ValueError, match="head W has shape"):
        U.Model(layers, (head[0][:-8], head[1], head[2]), s.hidden, s.q_out, s.kv_out, s.inter,
                s.vocab, s.r)


class _FakeCuda:
    """Stands in for a contiguous CUDA tensor on device `cuda:<i>` (no GPU here)."""

    def __init__(self, index):
        self.is_cuda = True
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True


def test_operands_on_two_devices_are_rejected():
    """The library launches on the current device; tensors on another device would be
    addressed from the wrong context, so the binding refuses mixed devices."""
    a, b = _FakeCuda(0), _FakeCuda(1)
    assert U._dev(a, None, _FakeCuda(0)) == torch.device("cuda", 0)
    with pytest.raises(ValueError, match="one device per call"):
        U._dev(a, b)


def test_stream_of_another_device_is_rejected():
    class _S:
        device = torch.device("cuda", 1)
        cuda_stream = 0
    with pytest.raises(ValueError, match="stream is on"):
        U._stream(_S(), torch.device("cuda", 0))
