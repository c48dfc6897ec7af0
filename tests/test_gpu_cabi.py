"""The C ABI driven from a C program (no Python on the path): it uploads x0,
runs the fused sampler, MDS, reconstruction and Eq. (6) through the raw
entry points on its own CUDA stream, and writes the results to files that are
compared here with the float64 oracle."""
import os
import subprocess

import numpy as np
import pytest

import synth
from oracle import mds as omds, schedule as osched, seam as oseam
from oracle.ddim import ddim_run as o_run
from tests.gpu_util import TOL_MAP, TOL_RECOVER, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"

C_PROG = r"""
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime_api.h>
#include "tdm.h"

#define CK(x) do { int s_ = (int)(x); if (s_ != 0) { fprintf(stderr, "%s -> %d\n", #x, s_); return 1; } } while (0)

static int dump(const char *path, const float *d, size_t n) {
    float *h = (float *)malloc(n * sizeof(float));
    FILE *f = fopen(path, "wb");
    if (!h || !f || cudaMemcpy(h, d, n * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
    fwrite(h, sizeof(float), n, f);
    fclose(f);
    free(h);
    return 0;
}

int main(int argc, char **argv) {
    const int C = 1, T = 4, B = 8, S = 10;
    const size_t n = (size_t)C * T * B;
    tdm_tiling t = {C, T, B, 12, 1, 0, B, 0, 0};
    tdm_ctx *ctx = NULL;
    tdm_schedule *sch = NULL;
    cudaStream_t st;
    float *x0, *maps, *coords, *rec, *disc, *hx0;
    uint32_t flags = 0;
    FILE *f;
    if (argc < 2) return 2;
    CK(cudaSetDevice(0));
    CK(cudaStreamCreate(&st));
    CK(tdm_ctx_create(&ctx, 0));
    CK(tdm_init_schedule(ctx, &sch, 1000, 1e-4, 0.02, NULL, S, 0.0));
    hx0 = (float *)malloc((size_t)C * T * 4096 * sizeof(float));
    f = fopen(argv[1], "rb");
    if (!hx0 || !f || fread(hx0, sizeof(float), (size_t)C * T * 4096, f) != (size_t)C * T * 4096) return 3;
    fclose(f);
    CK(cudaMalloc((void **)&x0, (size_t)C * T * 4096 * sizeof(float)));
    CK(cudaMalloc((void **)&maps, n * 4096 * sizeof(float)));
    CK(cudaMalloc((void **)&coords, n * 192 * sizeof(float)));
    CK(cudaMalloc((void **)&rec, n * 4096 * sizeof(float)));
    CK(cudaMalloc((void **)&disc, (size_t)C * (T - 1) * sizeof(float)));
    CK(cudaMemcpyAsync(x0, hx0, (size_t)C * T * 4096 * sizeof(float), cudaMemcpyHostToDevice, st));
    CK(tdm_ddim_run(ctx, sch, maps, x0, 1.0f, 0.1f, 0.3f, 7u, 1, &t, st));
    CK(tdm_mds_recover(ctx, maps, (int64_t)n, coords, NULL, st));
    CK(tdm_pairwise_dist(ctx, coords, (int64_t)n, rec, st));
    CK(tdm_seam_discrepancy(ctx, rec, &t, disc, st));
    CK(tdm_ctx_sync(ctx, st, &flags));
    if (dump("maps.bin", maps, n * 4096) || dump("rec.bin", rec, n * 4096) || dump("disc.bin", disc, C * (T - 1)))
        return 4;
    tdm_schedule_destroy(sch);
    tdm_ctx_destroy(ctx);
    cudaFree(x0); cudaFree(maps); cudaFree(coords); cudaFree(rec); cudaFree(disc);
    cudaStreamDestroy(st);
    free(hx0);
    printf("ok %u\n", flags);
    return 0;
}
"""


def test_c_program_runs_the_pipeline(tmp_path):
    src = tmp_path / "pipeline.c"
    src.write_text(C_PROG)
    exe = tmp_path / "pipeline"
    libdir = os.path.join(ROOT, "tiled_distance_maps_b200")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
                    f"{CUDA}/include", str(src), "-o", str(exe), "-L", libdir, "-ltdm", f"-Wl,-rpath,{libdir}",
                    "-L", f"{CUDA}/lib64", "-lcudart", f"-Wl,-rpath,{CUDA}/lib64"], check=True)
    x0 = synth.chain_x0(2, 1, 4)
    (tmp_path / "x0.bin").write_bytes(np.ascontiguousarray(x0, dtype=np.float32).tobytes())
    out = subprocess.run([str(exe), str(tmp_path / "x0.bin")], capture_output=True, text=True, cwd=tmp_path)
    assert out.returncode == 0 and out.stdout.startswith("ok 0"), out
    maps = np.fromfile(tmp_path / "maps.bin", dtype=np.float32).astype(np.float64).reshape(1, 4, 8, 64, 64)
    ref = o_run(x0, osched.Schedule(S=10), 1.0, 0.1, 0.3, 7, np.arange(8), 8)
    e = (np.abs(maps - ref).max(axis=(-1, -2)) / np.abs(ref).max(axis=(-1, -2))).max()
    assert e <= TOL_MAP, e
    rec = np.fromfile(tmp_path / "rec.bin", dtype=np.float32).astype(np.float64).reshape(-1, 64, 64)
    Ro = omds.pairwise_distances(omds.classical_mds(ref.reshape(-1, 64, 64))[0])
    er = (np.abs(rec - Ro).max(axis=(-1, -2)) / np.abs(Ro).max(axis=(-1, -2))).max()
    assert er <= TOL_RECOVER, er
    disc = np.fromfile(tmp_path / "disc.bin", dtype=np.float32).astype(np.float64)
    d_ref = oseam.seam_discrepancy(Ro.reshape(1, 4, 8, 64, 64)).ravel()
    assert np.all(np.abs(disc - d_ref) <= 2.0 * np.abs(rec - Ro).max() + 1e-6)
