"""The quantized weight file: save_quantized / load_quantized round-trip every
byte of a single tensor and of a fused weight, and a file whose fields
disagree with one another is refused before anything is returned."""
import pytest
import torch

import nvfp4_w4a4_quantized_09_b200 as nv


def _bytes(n, seed):
    return torch.randint(0, 256, (n,), dtype=torch.uint8, generator=torch.Generator().manual_seed(seed))


def _single(rows=200, cols=96, layout=nv.SF_TCGEN05):
    return nv.QuantizedTensor(_bytes(rows * cols // 2, 1).reshape(rows, cols // 2),
                              _bytes(nv.sf_bytes(rows, cols, layout), 2),
                              torch.tensor([0.0123], dtype=torch.float32), rows, cols, layout)


def _fused(sizes=(64, 32, 32), cols=256):
    rows = sum(sizes)
    gs = [torch.tensor([v], dtype=torch.float32) for v in (0.02, 0.2, 0.002)[:len(sizes)]]
    return nv.FusedWeight(_bytes(rows * cols // 2, 3).reshape(rows, cols // 2),
                          _bytes(nv.sf_bytes(rows, cols), 4), gs, list(sizes), cols)


@pytest.mark.parametrize("layout", [nv.SF_TCGEN05, nv.SF_LINEAR])
def test_single_tensor_round_trip(tmp_path, layout):
    q = _single(layout=layout)
    nv.save_quantized(str(tmp_path / "w.pt"), q)
    r = nv.load_quantized(str(tmp_path / "w.pt"), device="cpu")
    assert isinstance(r, nv.QuantizedTensor)
    assert (r.rows, r.cols, r.layout) == (q.rows, q.cols, q.layout)
    assert torch.equal(r.codes, q.codes) and torch.equal(r.sf, q.sf)
    assert r.g.dtype == torch.float32 and r.g.tolist() == q.g.tolist()


def test_fused_weight_round_trip(tmp_path):
    w = _fused()
    nv.save_quantized(str(tmp_path / "f.pt"), w)
    r = nv.load_quantized(str(tmp_path / "f.pt"), device="cpu")
    assert isinstance(r, nv.FusedWeight)
    assert r.sizes == w.sizes and r.cols == w.cols and r.rows == w.rows
    assert torch.equal(r.codes, w.codes) and torch.equal(r.sf, w.sf)
    assert [g.item() for g in r.g_list] == [g.item() for g in w.g_list]
    assert [(o, n) for o, n, _ in r.segments()] == [(o, n) for o, n, _ in w.segments()]


def _tamper(tmp_path, **change):
    w = _fused()
    p = str(tmp_path / "t.pt")
    nv.save_quantized(p, w)
    d = torch.load(p, weights_only=True)
    d.update(change)
    torch.save(d, p)
    return p


@pytest.mark.parametrize("change,match", [
    (dict(format="something-else"), "not an nvfp4-w4a4"),
    (dict(version=2), "not an nvfp4-w4a4"),
    (dict(sizes=[64, 32, 16]), "inconsistent header"),
    (dict(cols=250), "inconsistent header"),
    (dict(layout=7), "inconsistent header"),
    (dict(sf=_bytes(100, 5)), "sf holds 100 bytes"),
    (dict(codes=_bytes(128 * 100, 6).reshape(128, 100)), r"codes must have shape \(128, 128\)"),
    (dict(g=torch.tensor([0.02, 0.2], dtype=torch.float32)), "g must hold at least 3"),
    (dict(g=torch.tensor([0.02, -0.2, 0.1], dtype=torch.float32)), "positive finite global scale"),
    (dict(g=torch.tensor([0.02, 0.2, 0.1], dtype=torch.float64)), "g must be a contiguous float32"),
])
def test_inconsistent_files_are_refused(tmp_path, change, match):
    with pytest.raises(ValueError, match=match):
        nv.load_quantized(_tamper(tmp_path, **change), device="cpu")


def test_extra_scale_bytes_are_refused(tmp_path):
    w = _fused()
    with pytest.raises(ValueError, match="scale bytes for a"):
        nv.load_quantized(_tamper(tmp_path, sf=torch.cat([w.sf, _bytes(512, 7)])), device="cpu")


def test_only_quantized_weights_are_saved(tmp_path):
    with pytest.raises(TypeError):
        nv.save_quantized(str(tmp_path / "x.pt"), torch.zeros(4))
