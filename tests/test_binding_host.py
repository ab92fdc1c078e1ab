"""The Python binding's argument checks, on the host: wrong dtypes, devices, shapes and
layouts are refused with ValueError before the C entry point is called."""
import pytest

torch = pytest.importorskip("torch")

import gqa_exact_attention_b200 as G  # noqa: E402


def _cpu(shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def test_fwd_refuses_host_tensors():
    q, k, v = _cpu((1, 8, 4, 64)), _cpu((1, 8, 2, 64)), _cpu((1, 8, 2, 64))
    with pytest.raises(ValueError):
        G.gqa_attn_fwd(q, k, v)


def test_fwd_refuses_wrong_dtype():
    q = _cpu((1, 8, 4, 64), torch.float16)
    with pytest.raises(ValueError):
        G.gqa_attn_fwd(q, _cpu((1, 8, 2, 64)), _cpu((1, 8, 2, 64)))


def test_kvcache_refuses_host_tensors_and_bad_lengths():
    q, k, v = _cpu((2, 1, 4, 64)), _cpu((2, 16, 2, 64)), _cpu((2, 16, 2, 64))
    with pytest.raises(ValueError):
        G.gqa_attn_fwd_kvcache(q, k, v)
    with pytest.raises(ValueError):
        G.gqa_attn_fwd_kvcache(q, k, v, cache_seqlens=torch.zeros(2, dtype=torch.int64))


def test_kvcache_refuses_mismatched_cache_shapes():
    q = _cpu((2, 1, 4, 64))
    with pytest.raises(ValueError):
        G.gqa_attn_fwd_kvcache(q, _cpu((2, 16, 2, 64)), _cpu((2, 8, 2, 64)))


def test_nvtx_ranges_only_when_asked(monkeypatch):
    calls = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: calls.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: calls.append(("pop",)))
    monkeypatch.delenv("GQA_NVTX", raising=False)
    with G._range("gqa_attn_fwd"):
        pass
    assert calls == []
    monkeypatch.setenv("GQA_NVTX", "0")
    with G._range("gqa_attn_fwd"):
        pass
    assert calls == []
    monkeypatch.setenv("GQA_NVTX", "1")
    with pytest.raises(RuntimeError):
        with G._range("gqa_attn_fwd_paged"):
            raise RuntimeError("a failed call still closes its range")
    assert calls == [("push", "gqa_attn_fwd_paged"), ("pop",)]
