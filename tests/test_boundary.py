"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every entry point the header declares, validates its arguments before any
CUDA call, and sizes its buffers as the pages' memory-cost table does."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mp():
    from load_balancing_plan_b200 import build
    build.build()
    from load_balancing_plan_b200 import moonep
    return moonep


def _declared():
    with open(os.path.join(ROOT, "include", "moonep.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moonep_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(mp):
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(mp.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mp.EXPORTS)


def test_version(mp):
    assert "sm_100a" in mp.version()


def _cfg(**kw):
    c = dict(R=4, L=4, S=64, K=2, H=128, B=4, C=128, C_max=128)
    c.update(kw)
    return c


@pytest.mark.parametrize("bad", [
    dict(R=0), dict(R=65), dict(L=0), dict(R=64, L=65), dict(K=0), dict(K=65),
    dict(H=12), dict(H=0), dict(B=-1), dict(B=1025), dict(C=127), dict(C_max=100),
    dict(S=-1, C=-2),
])
def test_bad_cfg_rejected(mp, bad):
    c = _cfg(**bad)
    with pytest.raises(mp.MoonepError) as ei:
        mp.moonep_ws_layout(c)
    assert ei.value.code == mp.ERR_ARG
    assert mp.last_error()
    assert mp._lib.moonep_plan_workspace_bytes(ctypes.byref(mp.cfg_of(c))) == 0
    with pytest.raises(mp.MoonepError) as ei:
        mp.moonep_plan(c, 16, 256, stream=0)
    assert ei.value.code == mp.ERR_ARG


def test_null_and_misaligned_pointers_rejected(mp):
    c = _cfg()
    for args in [(None, 256), (16, None), (16, 258), (18, 256)]:
        with pytest.raises(mp.MoonepError) as ei:
            mp.moonep_plan(c, *args, stream=0)
        assert ei.value.code == mp.ERR_ARG
    with pytest.raises(mp.MoonepError):
        mp.moonep_dispatch(c, 256, 8, 16, 256, 16, stream=0)      # x misaligned
    with pytest.raises(mp.MoonepError):
        mp.moonep_combine(c, 256, 256, 16, 16, 264, stream=0)     # out misaligned
    with pytest.raises(mp.MoonepError):
        mp.moonep_prefetch(c, 256, 256, 256, 12, stream=0)        # elems not a multiple of 8
    with pytest.raises(mp.MoonepError):
        mp.moonep_reduce_grad(c, 256, 256, 256, 6, stream=0)      # elems not a multiple of 4
    with pytest.raises(mp.MoonepError):
        mp.moonep_set_wait_limit(-1)


def test_layout_is_consistent(mp):
    for c in [_cfg(), dict(R=8, L=32, S=8192, K=8, H=7168, B=32, C=65536, C_max=65536),
              dict(R=16, L=24, S=2048, K=8, H=7168, B=4, C=16384, C_max=20480),
              _cfg(S=0, C=0, C_max=0), _cfg(B=0)]:
        lay = mp.moonep_ws_layout(c)
        tables = [k for k in mp.LAYOUT_FIELDS[3:] if k not in ("tables_end", "base", "n_blocks", "blk")]
        offs = sorted(lay[k] for k in tables)
        assert len(set(offs)) == len(offs)                      # every table has its own place
        assert offs[0] == lay["cnt"] == mp.WS_HEADER_WORDS and offs[-1] < lay["tables_end"]
        assert lay["tables_end"] == lay["base"] <= lay["words"]
        assert lay["words"] % 4 == 0
        T = c["R"] * c["S"]
        N = c["R"] * c["L"]
        # whole waves of 296 ranges of about 4 tokens, at most 2^22 / N
        # entries per expert (T itself if fewer); blocks of consecutive
        # ranges, at most 147 (one per counting CTA: all SMs but the planner's)
        w = max(1, min((T + 592) // 1184, (1 << 22) // (N * 296)))
        Q = min(T, 296 * w)
        assert lay["n_ranges"] == mp.moonep_num_ranges(T, N) == Q
        assert lay["n_blocks"] == min(Q, 147)
        assert lay["blk"] == lay["base"] + N * max(Q, 1)
        assert lay["words"] >= lay["blk"] + N * max(lay["n_blocks"], 1)
        assert mp.moonep_plan_workspace_bytes(c) == 4 * lay["words"]


def _memory_table():
    rows = {}
    with open(os.path.join(ROOT, "tests", "golden", "memory_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            if "=" in line:
                setup = dict(kv.split("=") for kv in line.split())
                continue
            mode, B, pre, red, disp, tot = line.split()
            rows[mode] = (int(B), float(pre), None if red == "none" else float(red), float(disp),
                          float(tot))
    return {k: int(v) for k, v in setup.items()}, rows


def test_rank_bytes_match_memory_table(mp):
    # "The Busiest Rank Sets Your Step Time", memory-cost table: per-rank
    # prefetch, gradient-reduce and dispatch buffers for S=4096, H=7168,
    # three projections of FFN size 2048, printed in GiB to two decimals
    setup, rows = _memory_table()
    S, K, H, I, P = setup["S"], setup["K"], setup["H"], setup["I"], setup["P"]
    gib = float(1 << 30)
    for mode, (B, pre, red, disp, tot) in rows.items():
        c = dict(R=8, L=32, S=S, K=K, H=H, B=B, C=S * K, C_max=S * K)
        rb = mp.moonep_rank_bytes(c, P * H * I)
        assert round(rb["prefetch_bytes"] / gib, 2) == pytest.approx(pre, abs=0.006)
        assert round(rb["dispatch_bytes"] / gib, 2) == pytest.approx(disp, abs=0.006)
        total = rb["prefetch_bytes"] + rb["dispatch_bytes"]
        if red is not None:
            assert round(rb["reduce_bytes"] / gib, 2) == pytest.approx(red, abs=0.006)
            total += rb["reduce_bytes"]
        assert round(total / gib, 2) == pytest.approx(tot, abs=0.006)


def test_plan_flags_checked_before_any_cuda_call(mp):
    c = _cfg()
    for flags in (0x4, -1, mp.PLAN_REMOTE_WEIGHTS | mp.PLAN_ONE_GROUP):
        with pytest.raises(mp.MoonepError) as ei:
            mp.moonep_plan_ex(c, flags, 16, 256, stream=0)
        assert ei.value.code == mp.ERR_ARG


def test_copy_out_arguments_checked_before_any_cuda_call(mp):
    c = _cfg()
    rows_bytes = c["R"] * c["C_max"] * c["H"] * 2
    for args in [(None, 256, 1 << 40), (256, 264, 1 << 40), (256, 1 << 40, 8),
                 (256, 4096, 4096 + rows_bytes - 16), (256, 4096 + 16, 4096)]:   # misaligned, overlapping
        with pytest.raises(mp.MoonepError) as ei:
            mp.moonep_copy_out(c, *args, stream=0)
        assert ei.value.code == mp.ERR_ARG


def test_view_generation_of_unknown_workspace_is_zero(mp):
    assert mp.moonep_view_generation(0x1000) == 0
    assert mp.moonep_view_generation(None) == 0


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "moonep.h"

int main(void) {
    moonep_cfg_t c = {8, 8, 4096, 8, 7168, 8, 32768, 32768};
    moonep_ws_layout_t lay;
    moonep_rank_bytes_t rb;
    if (moonep_ws_layout(&c, &lay) != MOONEP_OK) return 1;
    if (moonep_plan_workspace_bytes(&c) != (size_t)lay.words * 4) return 2;
    if (moonep_num_ranges(32768, 64) != lay.n_ranges) return 3;
    if (moonep_rank_bytes(&c, 2 * 7168 * 2048, &rb) != MOONEP_OK) return 4;
    if (rb.dispatch_bytes != (int64_t)32768 * 7168 * 2) return 5;
    if (moonep_set_wait_limit(-1) != MOONEP_ERR_ARG || strlen(moonep_last_error()) == 0) return 6;
    if (moonep_set_wait_limit(1 << 22) != MOONEP_OK) return 7;
    c.C = 1;  /* C must equal S*K */
    if (moonep_plan(&c, (const int32_t *)16, (void *)256, 0) != MOONEP_ERR_ARG) return 8;
    if (moonep_view_generation((void *)4096) != 0) return 9;
    printf("%s\n", moonep_version());
    return 0;
}
"""


def test_header_is_plain_c_and_links(mp, tmp_path):
    # the boundary is a C ABI: a C99 program that includes the header builds
    # against the library and calls its host-side entry points
    import subprocess
    src = tmp_path / "use_moonep.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_moonep"
    libdir = os.path.dirname(mp.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), "-L", libdir, "-lmoonep", "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert "sm_100a" in out.stdout
    # and as C++ (the header's extern "C" block)
    exe2 = tmp_path / "use_moonep_cpp"
    subprocess.check_call(["g++", "-std=c++17", "-x", "c++", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe2), "-L", libdir, "-lmoonep", "-Wl,-rpath," + libdir])
    assert subprocess.run([str(exe2)], capture_output=True).returncode == 0


C_GPU_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "moonep.h"

#define CHECK(x) do { if ((x) != 0) { printf("failed: %s (%s)\n", #x, moonep_last_error()); return 1; } } while (0)

int main(void) {
    /* R=4 ranks, L=4 experts each, S=64 tokens, K=2, H=128, B=4 slots */
    moonep_cfg_t c = {4, 4, 64, 2, 128, 4, 128, 256};
    const int R = 4, N = 16, T = 256, K = 2, H = 128;
    const int Cm = c.C_max;
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * T * K);
    uint16_t *x = (uint16_t *)malloc(2 * (size_t)T * H);
    uint16_t *recv = (uint16_t *)malloc(2 * (size_t)R * Cm * H);
    int32_t *dest = (int32_t *)malloc(sizeof(int32_t) * T * K);
    char *used;
    int t, k, h, g;
    for (t = 0; t < T; ++t) {
        /* expert 0 is hot: every even token routes to it */
        ids[t * K] = (t % 2 == 0) ? 0 : t % N;
        ids[t * K + 1] = (ids[t * K] + 1 + t % 3) % N;
        for (h = 0; h < H; ++h) x[t * H + h] = (uint16_t)((t * 131 + h * 7) & 0x3FFF);
    }
    size_t wsb = moonep_plan_workspace_bytes(&c);
    void *d_ws, *d_ids, *d_x, *d_recv, *d_dest;
    CHECK(cudaMalloc(&d_ws, wsb));
    CHECK(cudaMalloc(&d_ids, sizeof(int32_t) * T * K));
    CHECK(cudaMalloc(&d_x, 2 * (size_t)T * H));
    CHECK(cudaMalloc(&d_recv, 2 * (size_t)R * Cm * H));
    CHECK(cudaMalloc(&d_dest, sizeof(int32_t) * T * K));
    CHECK(cudaMemcpy(d_ids, ids, sizeof(int32_t) * T * K, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(d_x, x, 2 * (size_t)T * H, cudaMemcpyHostToDevice));
    CHECK(moonep_plan(&c, (const int32_t *)d_ids, d_ws, 0));
    CHECK(moonep_dispatch(&c, d_ws, d_x, (const int32_t *)d_ids, d_recv, (int32_t *)d_dest, 0));
    moonep_plan_info_t info;
    CHECK(moonep_plan_read(&c, d_ws, &info, NULL, 0));
    if (info.status & MOONEP_ST_ERROR_MASK) { printf("status %x\n", info.status); return 2; }
    if (info.n_replicas < 1) { printf("no replicas\n"); return 3; }
    CHECK(cudaMemcpy(recv, d_recv, 2 * (size_t)R * Cm * H, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(dest, d_dest, sizeof(int32_t) * T * K, cudaMemcpyDeviceToHost));
    used = (char *)calloc((size_t)R * Cm, 1);
    for (g = 0; g < T * K; ++g) {
        int d = dest[g];
        if (d < 0 || d >= R * Cm || used[d]) { printf("bad dest %d at %d\n", d, g); return 4; }
        used[d] = 1;
        if (memcmp(recv + (size_t)d * H, x + (size_t)(g / K) * H, 2 * (size_t)H) != 0) {
            printf("row %d differs\n", d);
            return 5;
        }
    }
    /* every rank holds exactly S*K rows below C (no fallback here) */
    for (t = 0; t < R; ++t) {
        int n = 0;
        for (k = 0; k < c.C; ++k) n += used[t * Cm + k];
        if (info.fallback_rows == 0 && n != c.C) { printf("rank %d holds %d rows\n", t, n); return 6; }
    }
    printf("ok replicas=%d migrated=%d\n", info.n_replicas, info.migrated_rows);
    return 0;
}
"""


@pytest.mark.gpu
def test_c_program_plans_and_dispatches_on_the_gpu(mp, tmp_path):
    # the library used from plain C with the CUDA runtime only (no PyTorch):
    # plan and dispatch on a skewed routing, rows checked on the host
    import subprocess
    src = tmp_path / "dispatch_c.c"
    src.write_text(C_GPU_PROGRAM)
    exe = tmp_path / "dispatch_c"
    libdir = os.path.dirname(mp.LIB_PATH)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-lmoonep", "-Wl,-rpath," + libdir,
                           "-L", os.path.join(cuda, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(cuda, "lib64")])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok")
