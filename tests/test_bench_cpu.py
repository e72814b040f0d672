"""CPU checks of bench.py's bookkeeping: the recorded DRAM traffic is reported
only while the kernel's sources match the digest stored with the capture."""
import bench


def _write(tmp_path, digest, value=123456):
    p = tmp_path / "traffic.txt"
    p.write_text("# a comment line: with a colon\n"
                 f"kernel: tc_dkdv\nworkload: w\ndram_bytes_per_launch: {value}\nsource_sha256: {digest}\n")
    return str(p)


def test_recorded_traffic_needs_matching_sources(tmp_path, monkeypatch):
    good = _write(tmp_path, bench.kernel_source_digest("tc_dkdv"))
    monkeypatch.setitem(bench.TRAFFIC_FILES, ("tc_dkdv", "w"), good)
    assert bench.recorded_traffic("tc_dkdv", "w") == 123456
    stale = _write(tmp_path, "0" * 64)
    monkeypatch.setitem(bench.TRAFFIC_FILES, ("tc_dkdv", "w"), stale)
    assert bench.recorded_traffic("tc_dkdv", "w") is None
    assert bench.recorded_traffic("tc_dq", "w") is None            # no capture recorded
    assert bench.recorded_traffic("tc_dkdv", "other") is None


def test_digest_covers_the_listed_sources():
    d = bench.kernel_source_digest("tc_dkdv")
    assert len(d) == 64 and d == bench.kernel_source_digest("tc_dkdv")
    assert "tc_bwd.cu" in bench.KERNEL_SOURCES["tc_dkdv"]


def test_committed_traffic_record_matches_the_current_sources():
    # the committed capture describes the kernel as it is in the tree
    assert bench.recorded_traffic("tc_dkdv", "causal_b1h32s32768d128_cp8_bf16") is not None


def test_merge_bytes_per_row():
    # read acc O + LSE, read part O + LSE, write acc O + LSE (fp32)
    assert bench.merge_bytes_per_row(128) == 1548
    assert bench.merge_bytes_per_row(64) == 3 * 64 * 4 + 12


def test_pre_bytes_per_row():
    # read O and dO rows (bf16) and LSE, write delta and LSE*log2(e)
    assert bench.pre_bytes_per_row(128) == 2 * 128 * 2 + 12
    assert bench.pre_bytes_per_row(64, 4) == 2 * 64 * 4 + 12


class _W:
    def __init__(self, B, H):
        self.B, self.H = B, H


def test_e2e_chunks_divide_the_heads_or_batch():
    assert bench.e2e_chunks(_W(1, 32), 4) == 4
    assert bench.e2e_chunks(_W(1, 6), 4) == 3       # largest divisor of 6 not above 4
    assert bench.e2e_chunks(_W(1, 2), 8) == 2
    assert bench.e2e_chunks(_W(2, 32), 4) == 2      # batch groups when B > 1
    assert bench.e2e_chunks(_W(1, 7), 1) == 1


def test_chunk_views_are_contiguous_and_cover_the_tensor():
    import torch
    for B, H in ((1, 8), (2, 4)):
        w = _W(B, H)
        c = bench.e2e_chunks(w, 4)
        for shape in ((B, H, 16, 8), (B, H, 16)):
            t = torch.arange(torch.Size(shape).numel()).reshape(shape)
            parts = bench.chunk_views(t, w, c)
            assert len(parts) == c
            assert all(p.is_contiguous() for p in parts)
            assert torch.equal(torch.cat(parts, dim=1 if B == 1 else 0), t)
            # views share the tensor's storage (copies into them land in place)
            assert all(p.untyped_storage().data_ptr() == t.untyped_storage().data_ptr() for p in parts)
