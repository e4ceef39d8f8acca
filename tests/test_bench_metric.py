"""The benchmark's algorithmic work figures, tied to the mask the oracle
implements: the forward counts 4·d FLOPs per visible (query, key) pair, the
decode counts every K/V cache row some query of the block can see exactly
once, plus q, out and lse."""
import bd_inputs
import bench
import oracle


def test_fwd_flops_training_shape_closed_form():
    # 4 · 128 · (2048² + 2048·32) · 4 · 32
    assert bench.fwd_flops(bd_inputs.FWD_TRAIN) == 279_172_874_240


def test_fwd_flops_counts_the_oracles_visible_pairs():
    lib = oracle.load()
    for (L, b) in [(12, 3), (16, 4), (10, 10), (9, 1)]:
        pairs = sum(oracle.fwd_sees(L, b, r, c, lib=lib)
                    for r in range(2 * L) for c in range(2 * L))
        s = bd_inputs.FwdShape("t", 2, 3, 1, L, b, 32)
        assert bench.fwd_flops(s) == 4 * s.d * pairs * s.B * s.Hq, (L, b)


def test_decode_bytes_count_each_visible_cache_row_once():
    lib = oracle.load()
    B, Hq, Hkv, b, d = 3, 4, 2, 5, 16
    lens = [0, 7, 20]
    for mode in (0, 1):
        s = bd_inputs.DecodeShape("t", B, Hq, Hkv, b, d, mode, 0, max(lens))
        rows = 0
        for n in lens:
            seen = {c for j in range(b) for c in range(n + b + 3)
                    if oracle.decode_sees(n, b, mode, j, c, lib=lib)}
            rows += len(seen)
        kv = rows * Hkv * d * 2 * 2          # K and V, bf16, once per kv-head
        qo = 2 * B * Hq * b * d * 2          # q read, out written, bf16
        lse = B * Hq * b * 4
        assert bench.decode_bytes(s, lens) == kv + qo + lse, mode


def test_decode_bytes_denoise_workload():
    s = bd_inputs.DEC_DENOISE
    assert bench.decode_bytes(s, [8192] * s.B) == 547_422_208


def test_traffic_is_quoted_only_for_the_kernel_sources_it_was_captured_on(monkeypatch):
    # a stored ncu traffic figure belongs to one digest of the kernel
    # sources; any other digest (the kernels changed since) quotes nothing
    nbytes, digest, _ = bench.TRAFFIC["bd_tc_pair_kernel"]
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    assert bench.traffic_of("bd_tc_pair_kernel") == nbytes
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "0" * 16)
    assert bench.traffic_of("bd_tc_pair_kernel") is None
    assert bench.traffic_of("no_such_kernel") is None


def test_kernel_source_digest_covers_every_listed_source():
    import os
    csrc = os.path.join(bench.ROOT, "block_diffusion_lm_attn_b200", "csrc")
    assert bench.KERNEL_SOURCES
    for name in bench.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(csrc, name)), name
    d = bench.kernel_source_digest()
    assert len(d) == 16 and int(d, 16) >= 0
