"""The memory-system probe (include/hashgrid_probe.h): argument checks on the host, and on
the GPU that each probe performs exactly the operations it reports, on the units its
pattern names (reductions of 1.0 into a zeroed buffer leave a total equal to the operations
times the values per operation, and the pair patterns put both lanes' units where the
pattern says)."""
import numpy as np
import pytest

import multiresolution_hash_grid_b200 as hg


@pytest.mark.parametrize("kind,width,pattern,nbytes,msg", [
    (3, 8, 0, 1 << 20, "kind"),
    (hg.HASHGRID_PROBE_RED_F16, 32, 0, 1 << 20, "width"),
    (hg.HASHGRID_PROBE_RED, 32, 0, 1 << 20, "width"),
    (hg.HASHGRID_PROBE_GATHER, 12, 0, 1 << 20, "width"),
    (hg.HASHGRID_PROBE_GATHER, 8, 9, 1 << 20, "pattern"),
    (hg.HASHGRID_PROBE_GATHER, 8, hg.HASHGRID_PROBE_SECTOR_PAIR, 1 << 20, "16-byte"),
    (hg.HASHGRID_PROBE_RED, 8, hg.HASHGRID_PROBE_LINE_PAIR, 1 << 20, "16-byte"),
    (hg.HASHGRID_PROBE_GATHER, 8, 0, 3000, "power of two"),
    (hg.HASHGRID_PROBE_GATHER, 8, 0, 128, "power of two"),
])
def test_probe_rejects_bad_arguments(kind, width, pattern, nbytes, msg):
    with pytest.raises(hg.HashGridError) as e:
        hg.hashgrid_probe(kind, width, pattern, 16, nbytes, 1000, 16, stream=0)
    assert e.value.code == hg.HASHGRID_ERR_ARG and msg in str(e.value)


def test_probe_rejects_non_device_buffer():
    with pytest.raises(hg.HashGridError) as e:
        hg.hashgrid_probe(hg.HASHGRID_PROBE_RED, 16, 0, 4096, 1 << 20, 1000, stream=0)
    assert e.value.code in (hg.HASHGRID_ERR_ARG, hg.HASHGRID_ERR_ALIGN)


PATTERNS = ["RANDOM", "XPAIR", "SECTOR_PAIR", "LINE_PAIR", "STREAM"]


@pytest.mark.gpu
@pytest.mark.parametrize("width", [4, 8, 16])
@pytest.mark.parametrize("pattern", PATTERNS)
def test_red_probe_adds_exactly_its_operations(width, pattern):
    torch = pytest.importorskip("torch")
    if pattern in ("SECTOR_PAIR", "LINE_PAIR") and width != 16:
        pytest.skip("pair patterns take 16-byte units")
    buf = torch.zeros(1 << 18, dtype=torch.float32, device="cuda")  # 1 MiB
    done = hg.hashgrid_probe(hg.HASHGRID_PROBE_RED, width, getattr(hg, f"HASHGRID_PROBE_{pattern}"), buf,
                             buf.numel() * 4, 1 << 20)
    torch.cuda.synchronize()
    assert done >= 1 << 20
    counts = buf.cpu().numpy().astype(np.float64)
    assert counts.sum() == done * (width // 4)   # every element count is an exact integer in fp32
    assert np.all(counts == np.round(counts))
    # each operation covers width/4 consecutive elements: a unit's elements agree
    units = counts.reshape(-1, width // 4)
    assert np.all(units == units[:, :1])
    if pattern == "STREAM":
        assert units.max() - units.min() <= 1   # a sweep covers every unit equally often (+-1)
    elif pattern == "SECTOR_PAIR":             # lanes 2k, 2k+1 hit both halves of a sector
        halves = units[:, 0].reshape(-1, 2)
        np.testing.assert_array_equal(halves[:, 0], halves[:, 1])
    elif pattern == "LINE_PAIR":               # first halves of sectors only, spread over the buffer
        assert np.all(units[1::2, 0] == 0)
        assert np.count_nonzero(units[0::2, 0]) > 0.9 * (units.shape[0] // 2)
    else:                                      # random units: spread over (nearly) all of them
        assert np.count_nonzero(units[:, 0]) > 0.9 * units.shape[0]


@pytest.mark.gpu
@pytest.mark.parametrize("width", [4, 8, 16])
@pytest.mark.parametrize("pattern", ["RANDOM", "XPAIR"])
def test_fp16_red_probe_adds_exactly_its_operations(width, pattern):
    torch = pytest.importorskip("torch")
    buf = torch.zeros(1 << 19, dtype=torch.float16, device="cuda")  # 1 MiB
    done = hg.hashgrid_probe(hg.HASHGRID_PROBE_RED_F16, width, getattr(hg, f"HASHGRID_PROBE_{pattern}"), buf,
                             buf.numel() * 2, 1 << 20)
    torch.cuda.synchronize()
    counts = buf.cpu().numpy().astype(np.float64)
    assert counts.max() <= 2048                 # integer counts stay exact in binary16
    assert counts.sum() == done * (width // 2)
    units = counts.reshape(-1, width // 2)
    assert np.all(units == units[:, :1])


@pytest.mark.gpu
@pytest.mark.parametrize("width", [4, 8, 16, 32])
@pytest.mark.parametrize("pattern", ["RANDOM", "XPAIR", "STREAM"])
def test_gather_probe_runs_and_writes_nothing(width, pattern):
    torch = pytest.importorskip("torch")
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    sink = torch.full((4,), 7.0, dtype=torch.float32, device="cuda")
    done = hg.hashgrid_probe(hg.HASHGRID_PROBE_GATHER, width, getattr(hg, f"HASHGRID_PROBE_{pattern}"), buf,
                             buf.numel(), 1 << 20, sink)
    torch.cuda.synchronize()
    assert done >= 1 << 20
    assert torch.all(buf == 0) and torch.all(sink == 7.0)
