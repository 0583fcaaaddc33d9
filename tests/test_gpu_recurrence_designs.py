"""Two ways to lay the selective-scan recurrence over a warp, measured on the same inputs.

The library's scan spreads a channel's d_state states over lanes and walks time
sequentially in every lane; the readout C.h of a step is a sum over lanes, done for 8
steps at a time by a butterfly transpose-reduce. The other layout spreads time over
lanes: a warp owns one (b, d) channel with all 16 states in each lane's registers, every
lane takes K consecutive steps of a 32 * K-step chunk, and the chunk is solved as an
associative scan of the per-lane maps h -> a h + b (a = exp(delta A), b = delta u B)
with warp shuffles, the chunk's end state carried in registers into the next chunk.

This test builds a standalone probe with nvcc that runs both recurrence cores (inputs
delta, delta*u, B, C already in fp32; the exps, the recurrence and the readout C.h in the
kernel) on the Mamba-130M layer shape (B 8, D 1536, L 2048, d_state 16), checks both
against a double-precision host recurrence on sampled channels, and prints the time of
each. Run with -s to see the figures.
"""
import os
import re
import subprocess

import pytest

pytestmark = pytest.mark.gpu

PROBE = r'''
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <cmath>
#include <vector>
#include <algorithm>
#include <cuda_runtime.h>

constexpr int N = 16;

__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// States over lanes: 8 lanes per channel, states 2j and 2j + 1 in lane j, time
// sequential. Each lane keeps its partial C.h of 8 steps; three butterfly levels leave
// the full sum of step t0 + j in lane j.
__global__ void __launch_bounds__(128) rec_states(const float* __restrict__ dl,
        const float* __restrict__ du, const float* __restrict__ Bm, const float* __restrict__ Cm,
        const float* __restrict__ A, float* __restrict__ y, int Dm, int L) {
    const int j = threadIdx.x & 7;
    const int ch = blockIdx.x * 16 + (threadIdx.x >> 3);
    const int b = ch / Dm, d = ch % Dm;
    const float a0 = A[d * N + 2 * j], a1 = A[d * N + 2 * j + 1];
    const float* dlr = dl + (size_t)ch * L;
    const float* dur = du + (size_t)ch * L;
    const float* Bb = Bm + (size_t)b * L * N + 2 * j;
    const float* Cb = Cm + (size_t)b * L * N + 2 * j;
    float* yr = y + (size_t)ch * L;
    float h0 = 0.f, h1 = 0.f;
    for (int t0 = 0; t0 < L; t0 += 8) {
        const float4 d0 = *reinterpret_cast<const float4*>(dlr + t0);
        const float4 d1 = *reinterpret_cast<const float4*>(dlr + t0 + 4);
        const float4 u0 = *reinterpret_cast<const float4*>(dur + t0);
        const float4 u1 = *reinterpret_cast<const float4*>(dur + t0 + 4);
        const float ds[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        const float us[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        float p[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float2 bb = *reinterpret_cast<const float2*>(Bb + (size_t)(t0 + u) * N);
            const float2 cc = *reinterpret_cast<const float2*>(Cb + (size_t)(t0 + u) * N);
            h0 = fmaf(ex2a(ds[u] * a0), h0, us[u] * bb.x);
            h1 = fmaf(ex2a(ds[u] * a1), h1, us[u] * bb.y);
            p[u] = fmaf(cc.x, h0, cc.y * h1);
        }
#pragma unroll
        for (int m = 4; m >= 1; m >>= 1) {
            const bool hi = (j & m) != 0;
#pragma unroll
            for (int i = 0; i < m; ++i) {
                const float send = hi ? p[i] : p[i + m];
                const float keep = hi ? p[i + m] : p[i];
                p[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        yr[t0 + j] = p[0];
    }
}

// Time over lanes: one warp per channel, all 16 states in each lane. Lane i takes steps
// c0 + i K .. c0 + i K + K - 1 of a 32 K-step chunk: it composes its K maps h -> a h + b
// into one, a Hillis-Steele scan over the lanes composes the maps of all earlier lanes
// (five shuffle rounds of an (a, b) pair per state), the chunk's incoming state enters
// through the exclusive prefix, and each lane then walks its K steps again to form h and
// C.h. STORE keeps the K steps' (a, b) in registers; otherwise the exps and B products
// are recomputed in the second walk.
template <int K, bool STORE>
__global__ void __launch_bounds__(128) rec_time(const float* __restrict__ dl,
        const float* __restrict__ du, const float* __restrict__ Bm, const float* __restrict__ Cm,
        const float* __restrict__ A, float* __restrict__ y, int Dm, int L) {
    const int lane = threadIdx.x & 31;
    const int ch = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int b = ch / Dm, d = ch % Dm;
    float a[N], carry[N];
#pragma unroll
    for (int n = 0; n < N; ++n) { a[n] = A[d * N + n]; carry[n] = 0.f; }
    const float* dlr = dl + (size_t)ch * L;
    const float* dur = du + (size_t)ch * L;
    float* yr = y + (size_t)ch * L;
    for (int c0 = 0; c0 < L; c0 += 32 * K) {
        const int t0 = c0 + lane * K;
        float ds[K], us[K];
#pragma unroll
        for (int k = 0; k < K; ++k) { ds[k] = dlr[t0 + k]; us[k] = dur[t0 + k]; }
        float ea[STORE ? K : 1][N], eb[STORE ? K : 1][N];
        float Ag[N], Bg[N];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const float4* Bt = reinterpret_cast<const float4*>(Bm + ((size_t)b * L + t0 + k) * N);
            float bv[N];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = Bt[q];
                bv[4 * q] = v.x; bv[4 * q + 1] = v.y; bv[4 * q + 2] = v.z; bv[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const float e = ex2a(ds[k] * a[n]), f = us[k] * bv[n];
                if (STORE) { ea[k][n] = e; eb[k][n] = f; }
                if (k == 0) { Ag[n] = e; Bg[n] = f; }
                else { Bg[n] = fmaf(e, Bg[n], f); Ag[n] *= e; }
            }
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
            for (int n = 0; n < N; ++n) {
                const float Ap = __shfl_up_sync(0xffffffffu, Ag[n], off);
                const float Bp = __shfl_up_sync(0xffffffffu, Bg[n], off);
                if (lane >= off) { Bg[n] = fmaf(Ag[n], Bp, Bg[n]); Ag[n] *= Ap; }
            }
        }
        float h[N];
#pragma unroll
        for (int n = 0; n < N; ++n) {
            float Ae = __shfl_up_sync(0xffffffffu, Ag[n], 1);
            float Be = __shfl_up_sync(0xffffffffu, Bg[n], 1);
            if (lane == 0) { Ae = 1.f; Be = 0.f; }
            h[n] = fmaf(Ae, carry[n], Be);
            const float Al = __shfl_sync(0xffffffffu, Ag[n], 31);
            const float Bl = __shfl_sync(0xffffffffu, Bg[n], 31);
            carry[n] = fmaf(Al, carry[n], Bl);
        }
        float ys[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const float4* Ct = reinterpret_cast<const float4*>(Cm + ((size_t)b * L + t0 + k) * N);
            const float4* Bt = reinterpret_cast<const float4*>(Bm + ((size_t)b * L + t0 + k) * N);
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 cv = Ct[q];
                const float c4[4] = {cv.x, cv.y, cv.z, cv.w};
                float b4[4] = {0.f, 0.f, 0.f, 0.f};
                if (!STORE) {
                    const float4 bv = Bt[q];
                    b4[0] = bv.x; b4[1] = bv.y; b4[2] = bv.z; b4[3] = bv.w;
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int n = 4 * q + r;
                    const float e = STORE ? ea[STORE ? k : 0][n] : ex2a(ds[k] * a[n]);
                    const float f = STORE ? eb[STORE ? k : 0][n] : us[k] * b4[r];
                    h[n] = fmaf(e, h[n], f);
                    acc = fmaf(c4[r], h[n], acc);
                }
            }
            ys[k] = acc;
        }
#pragma unroll
        for (int k = 0; k < K; ++k) yr[t0 + k] = ys[k];
    }
}

static uint64_t rng = 0x9E3779B97F4A7C15ull;
static double urand() {                   // splitmix64 -> [0, 1)
    uint64_t z = (rng += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    return (z >> 11) * (1.0 / 9007199254740992.0);
}
static double nrand() { return sqrt(-2.0 * log(urand() + 1e-300)) * cos(6.283185307179586 * urand()); }

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { printf("cuda %s\n", cudaGetErrorString(e_)); return 1; } } while (0)

int main() {
    const int Bn = 8, Dm = 1536, L = 2048, rows = Bn * Dm;
    const size_t nx = (size_t)rows * L, nbc = (size_t)Bn * L * N;
    std::vector<float> dl(nx), du(nx), Bh(nbc), Ch(nbc), A(Dm * N);
    for (size_t i = 0; i < nx; ++i) {
        dl[i] = (float)exp(log(1e-3) + (log(1e-1) - log(1e-3)) * urand());   // delta
        du[i] = dl[i] * (float)nrand();                                       // delta * u
    }
    for (size_t i = 0; i < nbc; ++i) { Bh[i] = (float)nrand(); Ch[i] = (float)nrand(); }
    for (int d = 0; d < Dm; ++d)
        for (int n = 0; n < N; ++n) A[d * N + n] = (float)(-(n + 1) * 1.4426950408889634);  // A log2(e)
    float *ddl, *ddu, *dB, *dC, *dA, *dy;
    CK(cudaMalloc(&ddl, nx * 4)); CK(cudaMalloc(&ddu, nx * 4)); CK(cudaMalloc(&dy, nx * 4));
    CK(cudaMalloc(&dB, nbc * 4)); CK(cudaMalloc(&dC, nbc * 4)); CK(cudaMalloc(&dA, Dm * N * 4));
    CK(cudaMemcpy(ddl, dl.data(), nx * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(ddu, du.data(), nx * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dB, Bh.data(), nbc * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dC, Ch.data(), nbc * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dA, A.data(), Dm * N * 4, cudaMemcpyHostToDevice));

    // host recurrence in double on sampled channels
    const int samples[6] = {0, 1, 777, 5000, 9001, rows - 1};
    std::vector<std::vector<double>> ref(6, std::vector<double>(L));
    double ss = 0; size_t cnt = 0;
    for (int s = 0; s < 6; ++s) {
        const int ch = samples[s], b = ch / Dm, d = ch % Dm;
        double h[N] = {0};
        for (int t = 0; t < L; ++t) {
            double acc = 0;
            for (int n = 0; n < N; ++n) {
                h[n] = exp2((double)dl[(size_t)ch * L + t] * A[d * N + n]) * h[n] +
                       (double)du[(size_t)ch * L + t] * Bh[((size_t)b * L + t) * N + n];
                acc += Ch[((size_t)b * L + t) * N + n] * h[n];
            }
            ref[s][t] = acc; ss += acc * acc; ++cnt;
        }
    }
    const double rms = sqrt(ss / cnt);
    std::vector<float> yh(nx);
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0)); CK(cudaEventCreate(&e1));
    auto run = [&](const char* name, auto launch) -> int {
        for (int w = 0; w < 3; ++w) launch();
        CK(cudaDeviceSynchronize());
        std::vector<float> ms;
        for (int r = 0; r < 7; ++r) {
            CK(cudaEventRecord(e0)); launch(); CK(cudaEventRecord(e1));
            CK(cudaEventSynchronize(e1));
            float m; CK(cudaEventElapsedTime(&m, e0, e1)); ms.push_back(m);
        }
        CK(cudaGetLastError());
        std::sort(ms.begin(), ms.end());
        CK(cudaMemcpy(yh.data(), dy, nx * 4, cudaMemcpyDeviceToHost));
        double err = 0;
        for (int s = 0; s < 6; ++s)
            for (int t = 0; t < L; ++t)
                err = std::max(err, fabs((double)yh[(size_t)samples[s] * L + t] - ref[s][t]));
        printf("design %s ms %.4f err_rms %.3e\n", name, ms[3], err / rms);
        CK(cudaMemset(dy, 0, nx * 4));
        return 0;
    };
    if (run("states_over_lanes", [&] { rec_states<<<rows / 16, 128>>>(ddl, ddu, dB, dC, dA, dy, Dm, L); })) return 1;
    if (run("time_over_lanes_K1", [&] { rec_time<1, true><<<rows / 4, 128>>>(ddl, ddu, dB, dC, dA, dy, Dm, L); })) return 1;
    if (run("time_over_lanes_K2", [&] { rec_time<2, true><<<rows / 4, 128>>>(ddl, ddu, dB, dC, dA, dy, Dm, L); })) return 1;
    if (run("time_over_lanes_K4_recompute", [&] { rec_time<4, false><<<rows / 4, 128>>>(ddl, ddu, dB, dC, dA, dy, Dm, L); })) return 1;
    printf("ex2_per_launch %.0f\n", (double)nx * N);
    return 0;
}
'''


def test_states_over_lanes_against_time_over_lanes(tmp_path):
    src = tmp_path / "recurrence_designs.cu"
    exe = tmp_path / "recurrence_designs"
    src.write_text(PROBE)
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)], text=True, timeout=600)
    print(out)
    rows = re.findall(r"^design (\S+) ms ([\d.]+) err_rms ([\d.e+-]+)$", out, re.M)
    assert len(rows) == 4, out
    for name, ms, err in rows:
        # fp32 recurrence with ex2.approx over 2048 steps against the double recurrence
        assert float(err) <= 1e-4, (name, err)
        assert float(ms) > 0
