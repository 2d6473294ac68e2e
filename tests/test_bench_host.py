"""Host-side pieces of bench.py (CPU only): the kernel-code hash that decides
whether the committed ncu traffic figures still describe the kernel, and the
algorithmic byte count of the roofline."""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

CSRC = os.path.join("recurrent_vision_backbone_chunkwise_b200", "csrc")


@pytest.fixture
def tree(tmp_path, monkeypatch):
    """A copy of the kernel sources and the profile summary, with bench.ROOT
    pointing at it."""
    os.makedirs(tmp_path / CSRC)
    for name in bench.KERNEL_FILES:
        shutil.copy(os.path.join(ROOT, CSRC, name), tmp_path / CSRC / name)
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(ROOT, "profiles", "gla_fused_kernel.md"), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def _edit(path, fn):
    with open(path) as f:
        text = f.read()
    with open(path, "w") as f:
        f.write(fn(text))


def test_code_hash_ignores_comments_and_whitespace(tree):
    h0 = bench.kernel_code_hash()
    _edit(tree / CSRC / "gla_fused.cu", lambda t: "// a new comment line\n" + t.replace("\n", "\n\n", 3))
    _edit(tree / CSRC / "sm100.cuh", lambda t: t + "\n/* trailing\n block comment */\n")
    assert bench.kernel_code_hash() == h0


@pytest.mark.parametrize("name", ["gla_fused.cu", "sm100.cuh"])
def test_code_hash_sees_code_changes(tree, name):
    h0 = bench.kernel_code_hash()
    _edit(tree / CSRC / name, lambda t: t + "\nconstexpr int kProbe = 1;\n")
    assert bench.kernel_code_hash() != h0


def test_traffic_only_while_the_profile_matches(tree):
    prof = tree / "profiles" / "gla_fused_kernel.md"
    _edit(prof, lambda t: "kernel_code_sha256_16: %s\n" % bench.kernel_code_hash() +
          t.replace("kernel_code_sha256_16", "earlier_hash"))
    got = bench.profiled_traffic("1024_b4")
    assert isinstance(got, int) and got > 0
    assert bench.profiled_traffic("no_such_workload") is None
    _edit(tree / CSRC / "gla_fused.cu", lambda t: t + "\nconstexpr int kProbe = 2;\n")
    assert bench.profiled_traffic("1024_b4") is None


def test_workload_bytes_per_token_head():
    """768 B per token-head at d = 64 in fp16 (q, k, v, out at 2 B per element,
    log_alpha at 4 B), plus the fp32 final state per (b,h)."""
    from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS, Shape

    shape, dtype = CONFIGS["640_b1"]
    assert bench.workload_bytes(shape, dtype) == 6 * 1600 * 768 + 6 * 64 * 64 * 4
    s = Shape(1, 1, 2, 3, 128, 64)  # d_k = 128, d_v = 64, fp32
    assert bench.workload_bytes(s, "f32") == 6 * (128 * 4 * 2 + 64 * 4 + 128 * 4 + 64 * 4) + 128 * 64 * 4


def test_tail_traffic_follows_its_own_code_hash(tmp_path, monkeypatch):
    """The output tail's profile is gated by the hash of its own sources, not
    by the attention kernel's."""
    os.makedirs(tmp_path / CSRC)
    for name in set(bench.TAIL_FILES) | set(bench.KERNEL_FILES):
        shutil.copy(os.path.join(ROOT, CSRC, name), tmp_path / CSRC / name)
    os.makedirs(tmp_path / "profiles")
    prof = "output_tail_kernel_1024_b4.md"
    shutil.copy(os.path.join(ROOT, "profiles", prof), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the copy names the current code's hash, as a fresh capture would
    _edit(tmp_path / "profiles" / prof,
          lambda t: "kernel_code_sha256_16: %s\n" % bench.kernel_code_hash(bench.TAIL_FILES) +
          t.replace("kernel_code_sha256_16", "earlier_hash"))
    got = bench.profiled_traffic("1024_b4", prof, bench.TAIL_FILES)
    assert isinstance(got, int) and got > 0
    _edit(tmp_path / CSRC / "gla_fused.cu", lambda t: t + "\nconstexpr int kProbe = 3;\n")
    assert bench.profiled_traffic("1024_b4", prof, bench.TAIL_FILES) == got
    _edit(tmp_path / CSRC / "output_tail.cu", lambda t: t + "\nconstexpr int kProbe = 4;\n")
    assert bench.profiled_traffic("1024_b4", prof, bench.TAIL_FILES) is None


def test_swiglu_widths_follow_the_attention_workload():
    """C = 64 channels per head of the workload, F = 4C, fp16 for the fp32 case."""
    assert bench.swiglu_shape("1024_b4") == (4, 64, 64, 768, 3072, "f16")
    assert bench.swiglu_shape("640_b1") == (1, 40, 40, 384, 1536, "f16")
    assert bench.swiglu_shape("tiny")[-1] == "f16"


def test_nvidia_smi_index_and_single_rank_group(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5,6")
    assert bench.smi_index(1) == 5
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1234")
    assert bench.smi_index(1) == 1
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.smi_index(3) == 3

    class One:
        world = 1

    assert bench.dist_setup(One(), None) is None
    bench.dist_barrier(None)  # a no-op without a group


def test_tokens_per_call_are_image_tokens():
    """tokens/s counts image tokens, B * grid_h * grid_w per call: every head
    of a token is processed by the same call and is not counted again."""
    from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS

    assert bench.image_tokens(CONFIGS["640_b1"][0]) == 1600
    assert bench.image_tokens(CONFIGS["1024_b4"][0]) == 4 * 4096
    assert bench.image_tokens(CONFIGS["16k_d128"][0]) == 16384


def test_both_arms_print_the_same_config():
    """The reference arm and the GPU arm describe a workload with one function,
    so their config objects are equal for every workload and world size."""
    for name in ("640_b1", "1024_b4", "16k_d64", "16k_d128"):
        for world in (1, 2):
            a, b = bench.workload_config(name, world), bench.workload_config(name, world)
            assert a == b and a["workload"] == name and a["tokens"] > 0
    assert set(bench.PER_CONFIG) == {"1024_b4", "16k_d64", "16k_d128"}
