"""Host logic of the benchmark that needs no GPU: workload selection,
per-mode byte accounting and kernel naming, and the traffic figure taken
from the committed ncu summary."""

import pytest

import bench


def _layout(*argv):
    return bench.make_layout(bench.parse_args(list(argv)))


def test_batch_sizes_each_workload():
    assert _layout("--batch", "64").num_seqs == 64
    spec = _layout("--config", "llama3_8b_spec4", "--batch", "64")
    assert spec.num_seqs == 64 and spec.q_len == 4
    assert _layout("--config", "llama7b", "--batch", "16").num_seqs == 16
    shared = _layout("--config", "llama2_70b_shared", "--batch", "64")
    assert shared.num_seqs == 64 and len(shared.share_groups) == 16
    with pytest.raises(SystemExit):
        _layout("--config", "llama2_70b_shared", "--batch", "62")  # 4 samples per prompt
    with pytest.raises(SystemExit):
        _layout("--config", "opt13b_long_b16", "--batch", "8")


def test_shared_prefix_counts_each_block_once():
    L = _layout("--config", "llama2_70b_shared", "--batch", "64")
    plain, shared = bench.step_bytes(L, "plain"), bench.step_bytes(L, "shared_prefix")
    assert shared["decode"] == shared["decode_unique_blocks"] < plain["decode"] == plain["decode_per_sequence"]
    # 16 prompts of 128 blocks shared by 4 samples: the per-sequence count reads
    # each shared block 4 times, the unique count once
    assert plain["decode"] - shared["decode"] >= 16 * 3 * 127 * L.num_kv_heads * 8192


def test_kernel_names_follow_the_mode():
    L = _layout("--config", "llama7b", "--batch", "16")
    assert "tcgen05" in bench.decode_kernel_name(L, "plain")
    assert "CUDA cores" in bench.decode_kernel_name(L, "cuda_cores")
    assert bench.decode_entry(L, "cuda_cores") == "pa_decode"
    spec = _layout("--config", "llama3_8b_spec4", "--batch", "64")
    assert "multi-query" in bench.decode_kernel_name(spec, "plain")
    assert bench.decode_entry(spec, "plain") == "pa_decode_multi"


def test_profiled_traffic_only_for_the_profiled_workload():
    import re

    full = _layout()
    traffic = bench.profiled_traffic(full)
    algorithmic = bench.step_bytes(full)["decode"]
    summary = open(bench.PROFILE_SUMMARY).read()
    taken_on = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", summary).group(1)
    if taken_on == bench.kernel_source_hash():
        # DRAM bytes of the profiled kernel sit just above the algorithmic bytes
        assert traffic is not None and algorithmic <= traffic < 1.05 * algorithmic
    else:
        assert traffic is None  # the kernel changed since the capture
    assert bench.profiled_traffic(full, "shared_prefix") is None
    assert bench.profiled_traffic(_layout("--batch", "64")) is None


def test_one_launch_form_and_its_bytes():
    """The step's new-token writes go inside the tensor-core decode launch
    for the decode workloads that write, not for the prefill kernel's
    workload or the CUDA-core kernel, nor without new tokens; that launch's
    algorithmic bytes add the new tokens' K/V read and written."""
    full = _layout()
    assert bench.one_launch_step(full, "plain", "one_launch")
    assert not bench.one_launch_step(full, "plain", "separate")
    assert not bench.one_launch_step(full, "cuda_cores", "one_launch")
    assert not bench.one_launch_step(_layout("--config", "llama3_8b_prefill256", "--batch", "16"), "plain",
                                     "one_launch")
    assert not bench.one_launch_step(_layout("--config", "llama7b", "--batch", "16"), "plain", "one_launch")
    b = bench.step_bytes(full)
    T = full.num_new_tokens
    assert b["write"] == T * full.num_kv_heads * full.head_dim * 2 * 2 * 2 + T * 8
    assert b["step"] == b["decode"] + b["write"] + b["copy"]


def test_implied_model_rate_uses_each_models_layer_count():
    assert bench.model_layers(_layout()) == ("llama3_8b", 32)
    assert bench.model_layers(_layout("--config", "llama2_70b_shared", "--batch", "64")) == ("llama2_70b", 80)
    assert bench.model_layers(_layout("--config", "opt13b_long_b8")) == ("opt13b", 40)
    assert bench.model_layers(_layout("--config", "tiny")) == (None, None)
