"""The C-ABI library loads and exports every entry point include/dec.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dec.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:int|const char\*)\s+(dec_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def lib():
    import persistent_sm_decode_02_b200 as pkg
    if not os.path.exists(pkg.LIB_PATH):
        import persistent_sm_decode_02_b200.build as b
        b.build()
    return ctypes.CDLL(pkg.LIB_PATH)


def test_header_declares_the_lifecycle():
    names = _declared()
    for n in ("dec_create", "dec_load_weights", "dec_set_kv_cache", "dec_step", "dec_reset", "dec_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared():
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    import persistent_sm_decode_02_b200.dec as d
    assert sorted(d.EXPORTED) == _declared()
    for n in _declared():
        assert callable(getattr(d, n))


def test_constants_match_header():
    import persistent_sm_decode_02_b200.dec as d
    src = open(HEADER).read()
    for name, val in re.findall(r"#define\s+(DEC_\w+)\s+\(?(-?\w+)\)?", src):
        if name == "DEC_H_":
            continue
        v = int(val.rstrip("u"), 0)
        if hasattr(d, name):
            assert getattr(d, name) == v, name
    enum = dict((k, int(v)) for k, v in re.findall(r"(DEC_W_\w+)\s*=\s*(\d+)", src))
    names = {"embed": "EMBED", "final_norm": "FINAL_NORM", "lm_head": "LM_HEAD", "attn_norm": "ATTN_NORM",
             "wq": "Q", "wk": "K", "wv": "V", "wo": "O", "ffn_norm": "FFN_NORM", "w_gate": "GATE", "w_up": "UP",
             "w_down": "DOWN", "q_a": "Q_A", "q_a_norm": "Q_A_NORM", "q_b": "Q_B", "kv_a": "KV_A",
             "kv_a_norm": "KV_A_NORM", "kv_b": "KV_B", "router": "ROUTER", "exp_gate": "EXP_GATE",
             "exp_up": "EXP_UP", "exp_down": "EXP_DOWN", "sh_gate": "SH_GATE", "sh_up": "SH_UP",
             "sh_down": "SH_DOWN"}
    for k, v in d.DEC_W.items():
        assert enum["DEC_W_" + names[k]] == v, k


def test_config_struct_matches_header_field_order():
    import persistent_sm_decode_02_b200.dec as d
    src = open(HEADER).read()
    body = src[src.index("typedef struct dec_config"):src.index("} dec_config;")]
    fields = []
    for line in body.splitlines()[1:]:
        line = line.split("/*")[0].strip().rstrip(";")
        if not line:
            continue
        _, rest = line.split(None, 1)
        fields += [f.strip() for f in rest.split(",")]
    assert [f[0] for f in d.dec_config._fields_] == fields
    assert ctypes.sizeof(d.dec_config) == 4 * len(fields)


def test_create_without_device_reports_an_error():
    """On a machine without a GPU dec_create fails cleanly with a CUDA error code, never aborts."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import persistent_sm_decode_02_b200 as pkg
    from synth import workloads
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(workloads.get("tiny_dense_f32")))
    assert e.value.code in (pkg.dec.DEC_ERR_CUDA, pkg.dec.DEC_ERR_UNSUPPORTED)


def test_invalid_config_is_rejected_before_any_device_call():
    import persistent_sm_decode_02_b200 as pkg
    from synth import workloads
    w = workloads.get("tiny_dense_f32", n_kv_heads=3)  # 4 heads not divisible by 3
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(w))
    assert e.value.code == pkg.dec.DEC_ERR_INVALID_ARG
    w = workloads.get("tiny_dense_f32", head_dim=96)
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(w))
    assert e.value.code == pkg.dec.DEC_ERR_UNSUPPORTED


@pytest.mark.parametrize("over", [
    dict(n_heads=256),                # the tensor-core MLA tile holds 128 heads
    dict(qk_rope=32),                 # 64-dim K chunks of [latent | rope key]
    dict(kv_lora=256),
    dict(weight_dtype="f32"),         # MLA runs on bf16 activations
])
def test_mla_limits_are_rejected_before_any_device_call(over):
    import persistent_sm_decode_02_b200 as pkg
    from synth import workloads
    w = workloads.get("small_mla_moe_fp8", **over)
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(w))
    assert e.value.code == pkg.dec.DEC_ERR_UNSUPPORTED


def test_gqa_group_above_eight_is_rejected():
    import persistent_sm_decode_02_b200 as pkg
    from synth import workloads
    w = workloads.get("small_dense_g8_bf16", n_heads=32)  # 32 / 2 = 16 query heads per kv head
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(w))
    assert e.value.code == pkg.dec.DEC_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", sorted(__import__("synth.workloads", fromlist=["WORKLOADS"]).WORKLOADS))
def test_every_named_workload_passes_validation(name):
    """Each workload's configuration is accepted by the library's checks: without a GPU,
    dec_create gets as far as its first device call and fails there, not at validation."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import persistent_sm_decode_02_b200 as pkg
    from synth import workloads
    with pytest.raises(pkg.DecError) as e:
        pkg.Decoder(pkg.config_from_workload(workloads.get(name)))
    assert e.value.code == pkg.dec.DEC_ERR_CUDA and "cudaSetDevice" in str(e.value)
