"""The seeded input generator: deterministic, integer-exact, with the value
recipes the workloads state.  CPU only."""
import torch

from workloads import configs as C
from workloads import synth


def test_pcg_hash_known_values():
    # reference outputs of the published pcg_hash (PCG-RXS-M-XS 32) for 0, 1, 2
    x = torch.tensor([0, 1, 2], dtype=torch.int64)
    got = [int(v) for v in synth.pcg_hash(x)]
    want = [synth.pcg_hash_int(i) for i in range(3)]
    assert got == want
    assert all(0 <= v < 2 ** 32 for v in got)
    assert len(set(got)) == 3


def test_rows_are_deterministic_and_position_addressable():
    wl = C.shrink(C.get("long"), [300, 300])
    a = C.k_rows(wl, 1, torch.arange(0, 300))
    b = C.k_rows(wl, 1, torch.tensor([5, 250, 17]))
    assert torch.equal(a[[5, 250, 17]], b)
    assert not torch.equal(C.k_rows(wl, 0, torch.arange(10)), C.k_rows(wl, 1, torch.arange(10)))
    assert not torch.equal(C.k_rows(wl, 0, torch.arange(10)), C.v_rows(wl, 0, torch.arange(10)))


def test_value_recipes():
    wl = C.shrink(C.get("tiny"), [4000])
    k = C.k_rows(wl, 0, torch.arange(4000)).float()
    assert abs(k.mean().item()) < 0.01 and abs(k.std().item() - 1) < 0.01
    ki = C.kidx_rows(wl, 0, torch.arange(4000)).float()
    assert ki.min() == -8 and ki.max() == 8 and torch.equal(ki, ki.round())
    qs = C.queries(C.shrink(C.get("prefill"), [100, 100], new_tokens=64))
    assert qs["q"].shape == (128, 6, 256) and qs["q_idx"].shape == (128, 8, 128)
    assert set(qs["w"].unique().tolist()) <= {0.5, 1.0, 2.0}
    assert qs["q_pos"][0] == 100 and qs["q_pos"][-1] == 163 and qs["q_seq"][-1] == 1


def test_spikes_shift_keys_along_one_direction():
    wl = C.shrink(C.get("long"), [2000])
    pos = torch.arange(2000)
    m = synth.spike_mask(wl.seed, 0, pos, 5)
    frac = m.float().mean().item()
    assert 0.03 < frac < 0.07
    u = synth.spike_direction(wl.seed, 0, 1).float()
    k = C.k_rows(wl, 0, pos).float()[:, 1]
    proj = k @ u
    assert proj[m].mean() > 2.5 and abs(proj[~m].mean()) < 0.2


def test_quarter_lengths_and_block_table():
    wl = C.get("quarter")
    assert len(wl.lengths) == 64
    assert all(16384 <= L + 1 <= 262144 + 1 for L in wl.lengths)
    small = C.shrink(wl, [100, 700, 64], page_perm=True)
    bt = C.block_table(small)
    used = bt[bt >= 0]
    assert sorted(used.tolist()) == list(range(small.num_pages()))
