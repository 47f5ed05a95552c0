"""Host logic of the host-fed stepper: the packed layout of one step's inputs (CPU only)."""
import torch

from paged_kv_cache_363_b200.runner import pack_layout


def test_fields_are_aligned_disjoint_and_in_order():
    ts = {"q": torch.zeros(3, 5, 7, dtype=torch.bfloat16), "new_k": torch.zeros(3, 2, 7, dtype=torch.bfloat16),
          "slot_mapping": torch.zeros(3, dtype=torch.int64), "cow_pairs": torch.zeros(0, 2, dtype=torch.int64),
          "block_tables": torch.zeros(3, 9, dtype=torch.int32), "context_lens": torch.zeros(3, dtype=torch.int32),
          "none": None}
    fields, end = pack_layout(ts)
    assert [f[0] for f in fields] == ["q", "new_k", "slot_mapping", "block_tables", "context_lens"]
    prev_end = 0
    for name, off, n, dt, shape in fields:
        assert off % 256 == 0 and off >= prev_end
        assert n == ts[name].numel() * ts[name].element_size()
        assert dt == ts[name].dtype and shape == tuple(ts[name].shape)
        prev_end = off + n
    assert end == prev_end


def test_views_into_a_packed_buffer_round_trip():
    g = torch.Generator().manual_seed(3)
    ts = {"a": torch.randn(4, 3, generator=g).to(torch.bfloat16), "b": torch.arange(5, dtype=torch.int64),
          "c": torch.arange(7, dtype=torch.int32) - 3, "d": torch.randn(2, 2, generator=g)}
    fields, end = pack_layout(ts)
    buf = torch.zeros(end, dtype=torch.uint8)
    views = {n: buf[o:o + k].view(dt).view(s) for n, o, k, dt, s in fields}
    for n, t in ts.items():
        views[n].copy_(t)
    for n, t in ts.items():
        assert torch.equal(buf[[f for f in fields if f[0] == n][0][1]:][:t.numel() * t.element_size()]
                           .view(t.dtype).view(t.shape), t)


def test_empty_inputs_pack_to_nothing():
    fields, end = pack_layout({"q": torch.zeros(0, 4), "x": None})
    assert fields == [] and end == 0
