"""CPU tests of bench.py's accounting: the split partials that enter the
roofline's algorithmic bytes (written_partials, for both split modes), the
no-reconstruction bound, and the link between the committed ncu record and
the decode kernel's sources (the traffic figure is reported only while they
match)."""
import numpy as np

import bench

# page payloads of the three tiers at P = 64 (16 + 64 row bytes)
PAYLOAD = [16 + 64 * 512, 16 + 64 * 196, 16 + 64 * 180]


def table(units):
    """CSR page table of units given as lists of page tiers."""
    indptr = np.zeros(len(units) + 1, np.int32)
    ids = []
    for u, tiers in enumerate(units):
        indptr[u + 1] = indptr[u] + len(tiers)
        ids += [(t << 30) | (len(ids) + k) for k, t in enumerate(tiers)]
    return indptr, np.array(ids, np.uint32)


def test_global_split_counts_one_partial_per_run_of_a_spread_unit():
    # two units of 4 T1 pages each, 4 runs: every run holds 2 pages of one
    # unit, so each unit is spread over 2 runs -> 2 partials each
    indptr, ids = table([[1] * 4, [1] * 4])
    assert bench.written_partials(indptr, ids, PAYLOAD, 4) == 4
    # 2 runs: each unit inside one run -> no partial
    assert bench.written_partials(indptr, ids, PAYLOAD, 2) == 0
    # 8 runs = 8 x 2 units: unit-aligned, each unit 4 runs -> 4 partials each
    assert bench.written_partials(indptr, ids, PAYLOAD, 16) == 16


def test_unit_aligned_split_gives_runs_in_proportion_to_cost():
    # S = 32 >= 8 U: unit 0 costs three times unit 1; B(u) = u + round(P(u)(S-U)/C)
    indptr, ids = table([[1] * 6, [1] * 2])
    S, U = 32, 2
    first = [0, 1 + round(6 * (S - U) / 8), S]
    want = sum(first[u + 1] - first[u] for u in range(U))
    assert bench.written_partials(indptr, ids, PAYLOAD, S) == want
    # an empty unit writes nothing
    indptr, ids = table([[1] * 6, []])
    n = bench.written_partials(indptr, ids, PAYLOAD, S)
    assert n == (1 + round(6 * (S - U) / 6)) - 0


def test_empty_store_writes_no_partial():
    indptr, ids = table([[], []])
    assert bench.written_partials(indptr, ids, PAYLOAD, 148) == 0


def test_no_reconstruction_bound_and_rebuilt_key_bytes(monkeypatch):
    rec = {"sm_store_bytes": 600_000, "dram_bytes_write": 4_000_000}
    monkeypatch.setattr(bench, "profile_record", lambda: rec)
    out = bench.no_reconstruction(algo_bytes=200_000_000, nparts=100, G=4, rows=32,
                                  tier_counts=[10, 1000, 24, 5])
    bound = 100 * 4 * 132 * 4 + 32 * 128 * 4 + 32 * 4 + 8 * 32 + 0.01 * 200_000_000
    assert out["bound_bytes"] == int(bound)
    assert out["ok"] is True
    assert out["rebuilt_keys_bytes"] == (1000 + 24) * 256
    rec["sm_store_bytes"] = int(bound) + 1
    assert bench.no_reconstruction(200_000_000, 100, 4, 32, [10, 1000, 24, 5])["ok"] is False


def test_decode_digest_covers_the_decode_blocks_only():
    text = ("struct Other {\n  int a;\n};\nstruct DecodeParams {\n  int x;\n};\n"
            "struct DecodeWs {\n  size_t b;\n};\n__host__ __device__ inline DecodeWs decode_ws() {\n"
            "  DecodeWs w;\n  return w;\n}\nstruct Later {\n  int z;\n};\n")
    blocks = bench._decode_blocks(text)
    assert "struct DecodeParams" in blocks and "int x;" in blocks and "return w;" in blocks
    assert "struct Other" not in blocks and "struct Later" not in blocks


def test_committed_profile_describes_the_current_decode_kernel():
    """The ncu record under profiles/ was taken on the decode sources as they
    are: a change to the decode kernel needs a new capture (until then the
    bench reports no traffic figure)."""
    rec = bench.profile_record()
    assert rec is not None, "decode sources changed since the committed ncu capture"
    assert rec["traffic_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    assert bench.profiled_traffic() == rec["traffic_bytes_per_launch"]
