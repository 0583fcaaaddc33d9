"""The per-SM pipe rates the benchmark's ALU roofline divides by, measured here.

bench.py reports the scans against 16 ex2 results per clock per SM (MUFU) and the
heads form against 128 FP32 lanes per SM. This test builds a standalone probe with
nvcc (one CTA of 32 warps per SM, eight independent dependency chains per thread,
cycles from clock64 in each CTA) and checks that the measured rates match those
constants. Run with -s to see the measured figures.
"""
import os
import re
import subprocess

import pytest

import bench

pytestmark = pytest.mark.gpu

PROBE = r'''
#include <cstdio>
#include <cuda_runtime.h>
__device__ __forceinline__ float ex2_(float x) { float y; asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x)); return y; }
__device__ __forceinline__ float fma_(float a, float b, float c) { float r; asm volatile("fma.rn.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c)); return r; }
template <int MODE> __global__ void k(long long* cyc, float* sink, int iters) {
    float x[8];
    for (int i = 0; i < 8; ++i) x[i] = -1e-3f * (threadIdx.x + i);
    __syncthreads();
    long long t0 = clock64();
    for (int it = 0; it < iters; ++it)
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = MODE == 0 ? ex2_(x[i]) - 1.0f : fma_(x[i], 0.999f, 1e-4f);
    __syncthreads();
    long long t1 = clock64();
    float s = 0.f;
    for (int i = 0; i < 8; ++i) s += x[i];
    if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
    if (s == 12345.f) sink[blockIdx.x] = s;
}
template <int MODE> double rate(int nsm) {
    long long* c; float* s; const int T = 1024, IT = 4096;
    cudaMalloc(&c, nsm * sizeof(long long)); cudaMalloc(&s, nsm * sizeof(float));
    k<MODE><<<nsm, T>>>(c, s, 64);
    k<MODE><<<nsm, T>>>(c, s, IT);
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    long long h[1024]; cudaMemcpy(h, c, nsm * sizeof(long long), cudaMemcpyDeviceToHost);
    double cyc = 0; for (int i = 0; i < nsm; ++i) cyc += h[i]; cyc /= nsm;
    cudaFree(c); cudaFree(s);
    return (double)T * IT * 8 / cyc;
}
int main() {
    int nsm = 0; cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
    printf("sms %d\nex2 %.3f\nffma %.3f\n", nsm, rate<0>(nsm), rate<1>(nsm));
    return 0;
}
'''


def test_mufu_ex2_and_fp32_rates_match_the_roofline_constants(tmp_path):
    src = tmp_path / "pipe_rates.cu"
    exe = tmp_path / "pipe_rates"
    src.write_text(PROBE)
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", str(exe),
                           str(src)])
    out = subprocess.check_output([str(exe)], text=True, timeout=120)
    got = dict(re.findall(r"^(\w+) ([\d.]+)$", out, re.M))
    ex2, ffma, sms = float(got["ex2"]), float(got["ffma"]), int(float(got["sms"]))
    print(f"SMs {sms}; ex2 results per clock per SM {ex2:.2f}; FFMA results per clock per SM {ffma:.1f}")
    assert sms == bench.N_SM
    assert abs(ex2 - bench.SFU_EX2_PER_CLK_PER_SM) <= 0.05 * bench.SFU_EX2_PER_CLK_PER_SM
    assert 0.9 * bench.FP32_LANES_PER_SM <= ffma <= 1.02 * bench.FP32_LANES_PER_SM
