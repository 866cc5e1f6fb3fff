"""bench.py's roofline arithmetic and profile lookup, on the CPU.

The algorithmic bytes are the denominators of every roofline fraction the
bench prints; these cases restate them from the tensor sizes of each workload
(q, k, v in and o out, beta, gamma, the state) and check the per-kernel
figures and the traffic lookup's guards."""

import json
import os

import pytest

import bench
from frame_wise_gated_b200 import synth


def tensor_bytes(cfg):
    return cfg.B * cfg.H * cfg.T * cfg.S * cfg.D * (2 if cfg.bf16 else 4)


@pytest.mark.parametrize("name", ["rollout60s_720p", "clip5s_720p", "sweep_d64", "sweep_d256"])
def test_step_bytes_plain(name):
    cfg = synth.CONFIGS[name]
    beta = cfg.B * cfg.H * cfg.T * cfg.S * 4
    gamma = cfg.B * cfg.H * cfg.T * 4
    state = 2 * cfg.B * cfg.H * cfg.D * cfg.D * 4  # state_in and state_out
    assert bench.algorithmic_bytes(cfg) == 4 * tensor_bytes(cfg) + beta + gamma + state


def test_step_bytes_rollout_value():
    # 1936 frame-heads x 3600 tokens x 128 channels x 2 bytes = 1.7842 GB per tensor
    cfg = synth.CONFIGS["rollout60s_720p"]
    assert tensor_bytes(cfg) == 1_784_217_600
    assert bench.algorithmic_bytes(cfg) == 7_166_853_696


def test_step_bytes_prologue_counts_both_outputs():
    cfg = synth.CONFIGS["prologue_bidir_720p"]
    plain = synth.CONFIGS["rollout60s_720p"]
    # raw q, k, v in; forward and reverse outputs: one more tensor than plain
    assert bench.algorithmic_bytes(cfg) - bench.algorithmic_bytes(plain) == tensor_bytes(cfg)


def test_phase_bytes():
    cfg = synth.CONFIGS["rollout60s_720p"]
    ph = bench.phase_bytes(cfg)
    beta = cfg.B * cfg.H * cfg.T * cfg.S * 4
    assert ph["contract"] == ph["contract_scan"] == 2 * tensor_bytes(cfg) + beta == 3_596_313_600
    assert ph["readout"] == 2 * tensor_bytes(cfg)
    cfg4 = synth.CONFIGS["prologue_bidir_720p"]
    assert bench.phase_bytes(cfg4)["readout"] == 3 * tensor_bytes(cfg4)  # Q in, two outputs


def test_backward_bytes():
    cfg = synth.CONFIGS["rollout60s_720p"]
    per_tensor = tensor_bytes(cfg)
    frames = cfg.B * cfg.H * cfg.T
    beta2 = 2 * frames * cfg.S * 4      # beta in, dbeta out
    gamma2 = 2 * frames * 4             # gamma in, dgamma out
    states = 3 * cfg.B * cfg.H * cfg.D * cfg.D * 4
    assert bench.backward_bytes(cfg) == 7 * per_tensor + beta2 + gamma2 + states


def test_traffic_lookup_guards(tmp_path, monkeypatch):
    # an entry is used only for its workload and only on the sources it was taken on
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.csrc_digest()
    (prof / "ncu_traffic.json").write_text(json.dumps({
        "contract_scan": {"workload": "rollout60s_720p", "csrc_sha": good,
                          "dram_bytes_per_launch": 123},
        "readout": {"workload": "rollout60s_720p", "csrc_sha": "0" * 16,
                    "dram_bytes_per_launch": 456}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_digest", lambda: good)
    assert bench.ncu_traffic("contract_scan", "rollout60s_720p") == 123
    assert bench.ncu_traffic("contract_scan", "clip5s_720p") is None
    assert bench.ncu_traffic("readout", "rollout60s_720p") is None   # other sources
    assert bench.ncu_traffic("contract", "rollout60s_720p") is None  # no entry


def test_committed_traffic_entries_are_well_formed():
    p = os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")
    d = json.load(open(p))
    for phase, ent in d.items():
        assert phase in bench.phase_bytes(synth.CONFIGS[ent["workload"]])
        assert ent["dram_bytes_per_launch"] == ent["dram_read"] + ent["dram_write"]
        assert len(ent["csrc_sha"]) == 16
