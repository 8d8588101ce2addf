"""Saving and reloading the packed output (host plumbing, no GPU).

[QAS-QA] "Как работает quantization-aware scaling в AWQ для защиты важных весов?"
§9: the quantized model is saved and loaded back for inference."""
import pytest
import torch

from awq_activation_aware_b200 import persist


def fake_result(N=48, K=256, bits=4, group=128, n_alpha=20, seed=0):
    g = torch.Generator().manual_seed(seed)
    per = 16 if bits == 2 else 8
    return {
        "codes": torch.randint(-2**31, 2**31 - 1, (N, K // per), generator=g, dtype=torch.int64).to(torch.int32),
        "scales": torch.rand((N, K // group), generator=g).to(torch.float16),
        "zeros": torch.randint(-40, 40, (N, K // group), generator=g).to(torch.float16),
        "s_best": torch.rand(K, generator=g) + 0.5,
        "best_idx": torch.tensor([7], dtype=torch.int32),
        "losses": torch.rand(n_alpha, generator=g),
        "a": torch.rand(K, generator=g),
        "extra": torch.zeros(3),                       # not part of the format: left out
    }


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 64), (2, 64)])
def test_round_trip_is_exact(tmp_path, bits, group):
    r = fake_result(bits=bits, group=group)
    al = torch.arange(20, dtype=torch.float32) / 20
    p = tmp_path / "layer.pt"
    persist.save_quantized(p, r, bits, group, zero_point=(bits != 3), alphas=al)
    back = persist.load_quantized(p)
    assert back["bits"] == bits and back["group_size"] == group and back["zero_point"] == (bits != 3)
    for k in ("codes", "scales", "zeros", "s_best", "best_idx", "losses", "a"):
        assert back[k].dtype == r[k].dtype
        assert torch.equal(back[k].view(torch.uint8), r[k].contiguous().view(torch.uint8)), k   # bit for bit
    assert torch.equal(back["alphas"], al)
    assert "extra" not in back


def test_optional_tensors_may_be_absent(tmp_path):
    r = {k: v for k, v in fake_result().items() if k in ("codes", "scales", "zeros", "s_best", "best_idx")}
    p = tmp_path / "min.pt"
    persist.save_quantized(p, r, 4, 128)
    back = persist.load_quantized(p)
    assert set(back) == {"codes", "scales", "zeros", "s_best", "best_idx", "bits", "group_size", "zero_point"}


def test_save_rejects_inconsistent_results(tmp_path):
    p = tmp_path / "bad.pt"
    r = fake_result()
    with pytest.raises(ValueError):
        persist.save_quantized(p, r, 2, 128)                       # 2-bit words hold 16 codes: shapes disagree
    with pytest.raises(ValueError):
        persist.save_quantized(p, r, 4, 32)                        # unsupported group size
    bad = dict(r, scales=r["scales"].float())
    with pytest.raises(ValueError):
        persist.save_quantized(p, bad, 4, 128)                     # scales are fp16
    bad = dict(r, zeros=r["zeros"][:, :1])
    with pytest.raises(ValueError):
        persist.save_quantized(p, bad, 4, 128)
    missing = {k: v for k, v in r.items() if k != "s_best"}
    with pytest.raises(ValueError):
        persist.save_quantized(p, missing, 4, 128)
    with pytest.raises(ValueError):
        persist.save_quantized(p, r, 4, 128, alphas=torch.zeros(19))   # grid and losses differ in length
    with pytest.raises(ValueError):
        persist.save_quantized(p, dict(r, best_idx=torch.tensor([20], dtype=torch.int32)), 4, 128)
    assert not p.exists()


def test_load_rejects_other_files(tmp_path):
    p = tmp_path / "other.pt"
    torch.save({"weights": torch.zeros(4)}, p)
    with pytest.raises(ValueError):
        persist.load_quantized(p)
    r = fake_result()
    persist.save_quantized(p, r, 4, 128)
    blob = torch.load(p, weights_only=True)
    blob["version"] = persist.VERSION + 1
    torch.save(blob, p)
    with pytest.raises(ValueError):
        persist.load_quantized(p)
    blob["version"] = persist.VERSION
    blob["tensors"]["codes"] = blob["tensors"]["codes"][:, :-1]
    torch.save(blob, p)
    with pytest.raises(ValueError):
        persist.load_quantized(p)
