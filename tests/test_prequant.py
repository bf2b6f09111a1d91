"""In-memory prequantization of a state dict's routed expert projections
("fireworks-prequant 0.1.0", Quick start and Formats): the name filter on
the CPU, and on the GPU the packed outputs compared with the oracle bit for
bit, with every other tensor passed through untouched."""
import numpy as np
import pytest
import torch

import workloads
from mxfp8_block_scaled_warp_b200 import prequant


def test_expert_name_filter():
    quantized = [
        "model.layers.3.mlp.experts.17.gate_proj.weight",
        "model.layers.0.mlp.experts.0.up_proj.weight",
        "layers.12.mlp.experts.63.down_proj.weight",
        "language_model.model.layers.1.mlp.experts.2.down_proj.weight",
    ]
    kept = [
        "model.layers.3.mlp.shared_experts.gate_proj.weight",
        "model.layers.3.mlp.gate.weight",
        "model.layers.3.self_attn.q_proj.weight",
        "model.layers.3.mlp.experts.17.gate_proj.bias",
        "model.layers.3.mlp.experts.17.gate_proj.weight_scale_inv",
        "model.layers.3.mlp.gate_proj.weight",
        "xlayers.1.mlp.experts.2.up_proj.weight",
        "model.embed_tokens.weight",
    ]
    assert all(prequant.is_expert_weight(n) for n in quantized)
    assert not any(prequant.is_expert_weight(n) for n in kept)


def _state(layers=2, experts=3, d=256, f=128):
    """A small synthetic MoE state: per layer, experts with gate/up [f, d] and
    down [d, f] (N(0, 0.02) bf16), plus tensors that must pass through."""
    st = {}
    seed = 6000
    for l in range(layers):
        p = f"model.layers.{l}"
        st[f"{p}.self_attn.q_proj.weight"] = workloads.normal_bf16((d, d), 0.02, seed); seed += 1
        st[f"{p}.mlp.gate.weight"] = workloads.normal_bf16((experts, d), 0.02, seed); seed += 1
        st[f"{p}.input_layernorm.weight"] = torch.ones(d, dtype=torch.float32)
        for e in range(experts):
            for proj, shape in (("gate_proj", (f, d)), ("up_proj", (f, d)), ("down_proj", (d, f))):
                st[f"{p}.mlp.experts.{e}.{proj}.weight"] = workloads.normal_bf16(shape, 0.02, seed); seed += 1
        st[f"{p}.mlp.shared_experts.up_proj.weight"] = workloads.normal_bf16((f, d), 0.02, seed); seed += 1
    return st


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["mxfp8", "nvfp4"])
def test_quantize_state_dict_against_oracle(fpq, orc, fmt):
    st = _state()
    out = prequant.quantize_state_dict(st, fmt=fmt, device="cuda")
    torch.cuda.synchronize()
    n_expert = 0
    for name, t in st.items():
        if not prequant.is_expert_weight(name):
            assert out[name] is t                        # passed through, same object
            continue
        n_expert += 1
        assert name in out                               # codes under the original name
        base = name[: -len("weight")]
        x = workloads.as_u16(t)
        w, s = out[base + "weight"], out[base + "weight_scale_inv"]
        if fmt == "mxfp8":
            oq, os_ = orc.quant_mxfp8(x)
            assert w.dtype == torch.float8_e4m3fn and s.dtype == torch.uint8
            assert np.array_equal(w.view(torch.uint8).cpu().numpy(), oq)
            assert np.array_equal(s.cpu().numpy(), os_)
        else:
            oq, os_, og = orc.quant_nvfp4(x)
            g = out[base + "weight_scale_2"]
            assert w.dtype == torch.uint8 and s.dtype == torch.float8_e4m3fn and g.dtype == torch.float32
            assert w.shape == (t.shape[0], t.shape[1] // 2)
            assert np.array_equal(w.cpu().numpy(), oq)
            assert np.array_equal(s.view(torch.uint8).cpu().numpy(), os_)
            assert np.array_equal(g.reshape(1).cpu().numpy().view(np.uint32),
                                  np.asarray(og, np.float32).reshape(1).view(np.uint32))
    assert n_expert == 2 * 3 * 3
    # key order: each expert weight replaced in place by its outputs
    keys = list(out)
    assert keys.index("model.layers.0.mlp.experts.0.gate_proj.weight") < \
        keys.index("model.layers.0.mlp.experts.0.gate_proj.weight_scale_inv") < \
        keys.index("model.layers.0.mlp.experts.0.up_proj.weight")


@pytest.mark.gpu
def test_quantize_state_dict_rejects_non_bf16_experts(fpq):
    st = {"model.layers.0.mlp.experts.0.gate_proj.weight": torch.zeros(128, 256, dtype=torch.float32)}
    with pytest.raises(TypeError):
        prequant.quantize_state_dict(st, fmt="mxfp8")
    with pytest.raises(ValueError):
        prequant.quantize_state_dict({}, fmt="int4")
