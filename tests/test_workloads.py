"""The seeded input recipe (host logic, no GPU): the peaked workloads spike
exactly the chosen keys, in either reading of the spike."""
import pytest
import torch

from long_context_attention_td_b200.workloads import WORKLOADS, make_inputs


def _spiked(mode):
    w = WORKLOADS["bf16_peaked_h8_d128_n1m"].with_(H=3, N=5000, spike_mode=mode)
    return w, make_inputs(w, "cpu"), make_inputs(w.with_(spikes=0), "cpu")


@pytest.mark.parametrize("mode", ["aligned", "scaled"])
def test_exactly_the_spiked_keys_change(mode):
    w, sp, base = _spiked(mode)
    assert torch.equal(sp["q"], base["q"]) and torch.equal(sp["v"], base["v"])
    changed = (sp["k"] != base["k"]).any(dim=-1)          # [B,H,N]
    assert changed.sum(dim=-1).eq(w.spikes).all()


def test_aligned_spikes_point_along_q_with_eight_times_the_norm():
    w, sp, base = _spiked("aligned")
    changed = (sp["k"] != base["k"]).any(dim=-1)
    for h in range(w.H):
        pos = changed[0, h].nonzero().flatten()
        k_new = sp["k"][0, h, pos].double()
        k_old = base["k"][0, h, pos].double()
        q = sp["q"][0, h, 0].double()
        cos = (k_new @ q) / (k_new.norm(dim=-1) * q.norm())
        assert torch.all(cos > 0.999)
        ratio = k_new.norm(dim=-1) / k_old.norm(dim=-1)
        assert torch.allclose(ratio, torch.full_like(ratio, 8.0), rtol=1e-2)


def test_scaled_spikes_are_eight_times_the_key():
    w, sp, base = _spiked("scaled")
    changed = (sp["k"] != base["k"]).any(dim=-1)
    k_new = sp["k"][changed].double()
    k_old = base["k"][changed].double()
    # 8x is exact in bf16 (a power of two) unless it overflows, which N(0,1)*0.5 never does
    assert torch.equal(k_new, 8.0 * k_old)


def test_spike_positions_depend_only_on_the_seed():
    w = WORKLOADS["bf16_peaked_h8_d128_n1m"].with_(H=2, N=3000)
    a = make_inputs(w, "cpu")["k"]
    b = make_inputs(w, "cpu")["k"]
    assert torch.equal(a, b)
    with pytest.raises(ValueError):
        make_inputs(w.with_(spike_mode="other"), "cpu")
