"""Host-side logic of bench.py: byte accounting, the max-over-ranks timing and the
rank rules of the reference arm, run as two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_of_the_workload():
    sb = bench.step_bytes()
    # clip [1,3,121,704,1280] bf16 read + [1,192,31,176,320] bf16 written
    assert sb["haar_fwd"] == 3 * 121 * 704 * 1280 * 2 + 192 * 31 * 176 * 320 * 2 == 1_324_646_400
    assert sb["haar_inv"] == sb["haar_fwd"]
    # 64 x 56320 tokens: 16 fp32 read + 1 int32 written = 68 bytes per token
    assert sb["fsq_encode"] == 64 * 56320 * 68 == sb["fsq_decode"]


def test_job_throughput_is_weak_scaling():
    assert bench.job_throughput(10 ** 9, 10, 1, 1000.0) == pytest.approx(10.0)
    assert bench.job_throughput(10 ** 9, 10, 4, 1000.0) == pytest.approx(40.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(10.0 + rank, "cpu")

        class A:
            steps, warmup = 1, 0
        # Ranks other than 0 leave the reference arm at once, without work.
        rc = bench.run_reference(A, rank, world) if rank != 0 else 0
        dist.barrier()
        out[rank] = (m, rc)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 11.0
    assert res[1][1] == 0


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5


def test_threaded_baseline_parts_are_the_whole_oracle_step():
    """The parts the threaded CPU baseline times (per channel window chunks, per latent grid)
    compute exactly the unsplit oracle step."""
    import numpy as np

    import oracle
    import synth
    x64 = synth.bf16_bits_to_f64(synth.smooth_field((1, 2, 13, 8, 16), seed=11))
    lat = synth.fsq_input(4)[:3, :, :96]
    w = synth.fsq_weight()
    parts = bench.oracle_step_parts(x64, lat, w, windows_per_part=1)
    assert len(parts) == 2 * 3 + 3  # per channel: windows 0-1 in the first chunk, then 2 and 3; 3 grids
    out = [f() for f in parts]
    y = oracle.haar_fwd(x64)
    xr = oracle.haar_inv(y, 13, 8, 16)
    C = 2
    for kind, *rest in out:
        if kind == "haar":
            c, f0, yc, xc = rest
            t0 = 0 if f0 == 0 else (f0 + 3) // 4
            np.testing.assert_allclose(yc[0], y[0, c::C, t0:t0 + yc.shape[2]], rtol=0, atol=1e-12)
            np.testing.assert_allclose(xc[0, 0], xr[0, c, f0:f0 + xc.shape[2]], rtol=0, atol=1e-12)
        else:
            g, idx, dec = rest
            ref_idx, _, _ = oracle.fsq_encode(lat[g:g + 1], w)
            assert np.array_equal(idx, ref_idx)
            np.testing.assert_array_equal(dec, oracle.fsq_decode(ref_idx, w)[0])


def test_recorded_traffic_only_for_the_current_kernel_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from the profiles row whose digest matches the kernel sources
    as they are; a row taken on other sources (or a missing file) gives null."""
    import shutil
    csrc = tmp_path / "haar_wavelet_patching_b200" / "csrc"
    csrc.mkdir(parents=True)
    for fn in bench.KERNEL_SOURCES["haar_fwd"]:
        shutil.copy(os.path.join(ROOT, "haar_wavelet_patching_b200", "csrc", fn), csrc / fn)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("haar_fwd") is None  # no profiles file
    digest = bench.kernel_source_digest("haar_fwd")
    (tmp_path / "profiles").mkdir()
    table = "| kernel | bytes | digest | note |\n|---|---|---|---|\n"
    (tmp_path / "profiles" / "dram_traffic.md").write_text(table + "| haar_fwd | 123456 | 0000000000000000 | old |\n")
    assert bench.recorded_traffic("haar_fwd") is None
    (tmp_path / "profiles" / "dram_traffic.md").write_text(table + f"| haar_fwd | 123456 | {digest} | current |\n")
    assert bench.recorded_traffic("haar_fwd") == 123456.0
    assert bench.recorded_traffic("haar_inv") is None  # a row names its kernel
    with open(csrc / "haar_tma.cu", "a") as f:  # any edit of a source the kernel is built from
        f.write("\n")
    assert bench.recorded_traffic("haar_fwd") is None


def test_earlier_traffic_is_labelled_with_both_digests(tmp_path, monkeypatch):
    """With no row for the current sources, the newest row of the kernel is shown apart from
    roofline.traffic, with its digest and the current one."""
    import shutil
    csrc = tmp_path / "haar_wavelet_patching_b200" / "csrc"
    csrc.mkdir(parents=True)
    for fn in bench.KERNEL_SOURCES["haar_fwd"]:
        shutil.copy(os.path.join(ROOT, "haar_wavelet_patching_b200", "csrc", fn), csrc / fn)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    table = "| kernel | bytes | digest | note |\n|---|---|---|---|\n"
    (tmp_path / "profiles" / "dram_traffic.md").write_text(table + "| haar_fwd | 777 | 00000000aaaaaaaa | old |\n")
    digest = bench.kernel_source_digest("haar_fwd")
    assert bench.recorded_traffic("haar_fwd") is None
    assert bench.earlier_traffic("haar_fwd") == {"bytes": 777.0, "digest": "00000000aaaaaaaa",
                                                 "current_digest": digest}
    (tmp_path / "profiles" / "dram_traffic.md").write_text(table + f"| haar_fwd | 888 | {digest} | now |\n")
    assert bench.earlier_traffic("haar_fwd") is None and bench.recorded_traffic("haar_fwd") == 888.0
