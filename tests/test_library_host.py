"""Host-side checks of libkvtc (no GPU needed): the C ABI loads and exports every entry
point the header declares, the library's calibration (its own Jacobi eigen-solver)
matches the oracle's, plan files round-trip, and invalid arguments are rejected."""

import numpy as np
import pytest

from bit_quantization_head_b200 import kvtc
from bit_quantization_head_b200 import synth
from oracle import calibration as ocal


@pytest.fixture(scope="module")
def L():
    return kvtc.lib()


def test_library_exports_every_header_entry_point(L):
    names = kvtc.header_entry_points()
    assert len(names) >= 18
    for n in names:
        assert hasattr(L, n), n
    assert L.kvtc_version() == 1


def _compare_plans(plan, units, rtol_M=1e-6):
    # Calibration parity: (r, b) identical; delta and inv_delta equal to rounding; M
    # (fp32, after sign canonicalisation) within 1e-6 of the oracle's fp64 M normwise
    # (max |dM| <= 1e-6 max |M|); measured differences are a few fp32 ulp (~3e-8).
    assert plan.shape["n_units"] == len(units)
    for u, ou in enumerate(units):
        info = plan.unit(u)
        assert (info["r"], info["b"]) == (ou["r"], ou["b"]), u
        assert info["delta"] == pytest.approx(ou["delta"], rel=1e-9)
        assert abs(np.float32(info["inv_delta"]).view(np.int32) - np.float32(ou["inv_delta"]).view(np.int32)) <= 1
        w, lam = plan.weights(u)
        assert np.allclose(w, ou["w"], rtol=1e-8, atol=1e-12 * ou["w"].max())
        assert np.allclose(lam, ou["lam"], rtol=1e-8, atol=1e-12 * ou["lam"].max())
        M = plan.matrix(u)
        assert np.abs(M - ou["M"]).max() <= rtol_M * np.abs(ou["M"]).max(), (u, np.abs(M - ou["M"]).max())
        assert info["distortion"] == pytest.approx(ou["D"], rel=1e-8)


def test_calibrate_matches_oracle_fixed_allocation_head1():
    w = synth.WORKLOADS["head1-fp32-1k"]
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=1, n_kv_heads=1, group=1, seed=w.seed, fixed_r=16, fixed_b=4)
    units = ocal.calibrate(k, v, q, 1, 1, bpd=0, seed=w.seed, fixed_r=16, fixed_b=4)
    _compare_plans(plan, units)


def test_calibrate_matches_oracle_c2_llama_layer_2bpd():
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=1, n_kv_heads=8, group=4, bpd=2.0, seed=w.seed)
    units = ocal.calibrate(k, v, q, 1, 8, bpd=2.0, seed=w.seed)
    _compare_plans(plan, units)
    mu, bits = plan.budget()
    assert bits <= 2.0 * 128 * 16
    assert mu == pytest.approx(units[0]["mu"], rel=1e-6)


@pytest.mark.parametrize("mode", ["kl", "mse"])
def test_calibrate_matches_oracle_multilayer_1bpd(mode):
    w = synth.scaled(synth.WORKLOADS["llama8b-32L-128k-1bpd"], n_layers=2, n_cal=256)
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=2, n_kv_heads=8, group=4, bpd=1.0, seed=w.seed,
                               weight_mode=kvtc.WEIGHTS_KL if mode == "kl" else kvtc.WEIGHTS_MSE)
    units = ocal.calibrate(k, v, q, 2, 8, bpd=1.0, seed=w.seed, weight_mode=mode)
    _compare_plans(plan, units)


def test_calibrate_damped_c2_matches_oracle_and_sits_between_bounds():
    # the pages' iterative C2 ("C2, across heads": damped update, five rounds) against
    # the oracle's restatement, on the two-layer 1-bpd pool
    w = synth.scaled(synth.WORKLOADS["llama8b-32L-128k-1bpd"], n_layers=2, n_cal=256)
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=2, n_kv_heads=8, group=4, bpd=1.0, seed=w.seed,
                               c2_mode=kvtc.C2_DAMPED)
    units = ocal.calibrate(k, v, q, 2, 8, bpd=1.0, seed=w.seed, c2_mode="damped")
    _compare_plans(plan, units)
    lag = ocal.calibrate(k, v, q, 2, 8, bpd=1.0, seed=w.seed)
    total = 1.0 * 128 * 32
    assert sum(u["r"] * u["b"] for u in units) <= total
    D_damped = sum(u["D"] for u in units)
    D_lagrange = sum(u["D"] for u in lag)
    per_unit = int(total) // 32
    D_equal = sum(ocal.distortion(u["w"], *ocal.c1(u["w"], per_unit)) for u in lag)
    # the damped level iteration reaches the water-filling point: within 2 % of the
    # Lagrangian solver's total distortion, and far below the equal split
    assert D_damped <= 1.02 * D_lagrange and D_damped < D_equal
    mu, _ = plan.budget()
    assert mu == pytest.approx(units[0]["mu"], rel=1e-12)


def test_calibration_times_are_reported_per_phase():
    w = synth.scaled(synth.WORKLOADS["llama8b-32L-128k-1bpd"], n_layers=2, n_cal=256)
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=2, n_kv_heads=8, group=4, bpd=1.0, seed=w.seed)
    stats_s, alloc_s = plan.calib_seconds()
    assert stats_s > 0.0 and alloc_s > 0.0
    assert stats_s + alloc_s < 120.0


def test_calibrate_keys_only_matches_oracle():
    # keys-only ("k-only" results): the allocation covers the key units, values raw
    w = synth.scaled(synth.WORKLOADS["llama8b-32L-128k-1bpd"], n_layers=2, n_cal=256)
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=2, n_kv_heads=8, group=4, bpd=1.0, seed=w.seed, k_only=True)
    units = ocal.calibrate(k, v, q, 2, 8, bpd=1.0, seed=w.seed, k_only=True)
    _compare_plans(plan, units)
    for u in range(1, 32, 2):
        info = plan.unit(u)
        assert (info["r"], info["b"]) == (128, kvtc.RAW_BITS)
        assert info["page_bytes"] == 32768
    assert sum(plan.unit(u)["r"] * plan.unit(u)["b"] for u in range(0, 32, 2)) <= 1.0 * 128 * 16


def test_plan_create_accepts_raw_value_units_only_as_values():
    rng = np.random.default_rng(8)
    M = [np.linalg.qr(rng.standard_normal((128, 128)))[0][:16].astype(np.float32), np.eye(128, dtype=np.float32)]
    kvtc.kvtc_plan_create(1, 1, 1, [16, 128], [2, 16], [0.1, 2.0 ** -24], M)
    with pytest.raises(kvtc.KvtcError):
        kvtc.kvtc_plan_create(1, 1, 1, [128, 16], [16, 2], [2.0 ** -24, 0.1], M[::-1])
    with pytest.raises(kvtc.KvtcError):
        kvtc.kvtc_plan_create(1, 1, 1, [16, 64], [2, 16], [0.1, 2.0 ** -24], [M[0], M[1][:64]])


def test_plan_save_load_round_trip(tmp_path):
    w = synth.WORKLOADS["head1-fp32-1k"]
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=1, n_kv_heads=1, group=1, seed=1, fixed_r=16, fixed_b=4)
    p = tmp_path / "plan.bin"
    plan.save(p)
    again = kvtc.kvtc_plan_load(p)
    for u in range(2):
        assert again.unit(u) == plan.unit(u)
        assert np.array_equal(again.matrix(u), plan.matrix(u))
        assert np.array_equal(again.weights(u)[0], plan.weights(u)[0])
    raw = bytearray(p.read_bytes())
    raw[8] = 99                     # version field
    bad = tmp_path / "bad.bin"
    bad.write_bytes(bytes(raw))
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_plan_load(bad)
    assert e.value.status == 6      # EVERSION
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_plan_load(tmp_path / "missing.bin")
    assert e.value.status == 7      # EIO


def test_plan_create_validates_and_sizes_the_cache():
    M = [np.eye(128, dtype=np.float32)[:r] for r in (16, 10, 128, 2)]
    plan = kvtc.kvtc_plan_create(1, 2, 4, [16, 10, 128, 2], [4, 2, 8, 3], [0.5, 0.25, 1.0, 2.0], M)
    assert [plan.unit(u)["page_bytes"] for u in range(4)] == [16 * 64, 16 * 20, 16 * 1024, 16 * 6]
    assert kvtc.kvtc_cache_bytes(plan, 10) == 10 * 16 * (64 + 20 + 1024 + 6)
    assert kvtc.kvtc_unit_pool_offset(plan, 2, 10) == 10 * 16 * (64 + 20)
    assert np.array_equal(plan.matrix(1), M[1])
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_plan_create(1, 1, 1, [3, 2], [4, 4], [1.0, 1.0], [np.zeros((3, 128)), np.zeros((2, 128))])
    assert e.value.status == 1
    with pytest.raises(kvtc.KvtcError):
        kvtc.kvtc_plan_create(1, 1, 1, [2, 2], [9, 4], [1.0, 1.0], [np.zeros((2, 128))] * 2)
    with pytest.raises(kvtc.KvtcError):
        plan.weights(0)             # imported plans carry no calibration weights


def test_calibrate_rejects_bad_arguments():
    k = np.zeros((1, 1, 8, 64), np.float32)
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_calibrate(k, k, None, n_layers=1, n_kv_heads=1, group=1, weight_mode=kvtc.WEIGHTS_MSE)
    assert e.value.status == 1      # head_dim must be 128
    k = np.random.default_rng(0).standard_normal((1, 2, 16, 128)).astype(np.float32)
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_calibrate(k, k, None, n_layers=1, n_kv_heads=2, group=1, bpd=0.01,
                            weight_mode=kvtc.WEIGHTS_MSE)
    assert e.value.status == 4      # EINFEASIBLE: below 4 bits per unit
    with pytest.raises(kvtc.KvtcError):
        kvtc.kvtc_calibrate(k, k, None, n_layers=1, n_kv_heads=2, group=1, fixed_r=3, fixed_b=2)


def test_hot_calls_require_an_uploaded_plan():
    M = [np.eye(128, dtype=np.float32)[:16]] * 2
    plan = kvtc.kvtc_plan_create(1, 1, 1, [16, 16], [2, 2], [1.0, 1.0], M)
    desc = kvtc.CacheDesc(16, 4, 16, 1, 1, 0)
    L = kvtc.lib()
    import ctypes as C
    st = L.kvtc_encode_append(plan.handle, C.byref(desc), 0, C.c_void_p(16), C.c_void_p(16), 1,
                              C.c_void_p(16), C.c_void_p(16), 1, None)
    assert st == 8                  # ESTATE
    st = L.kvtc_decode_attention(plan.handle, C.byref(desc), 0, C.c_void_p(16), 1, C.c_void_p(16), 128, 0.0,
                                 C.c_void_p(16), 1, C.c_void_p(16), 1 << 20, None)
    assert st == 8
    assert b"upload" in L.kvtc_last_error()
    assert L.kvtc_decode_workspace_bytes(plan.handle, 1, 1024) > 0
