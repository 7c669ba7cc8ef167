// Epsilon-bar tile statistics (HiFA4 abstract: every measured attention tile
// shows a net loss of probability mass when P is quantized, median
// epsilon_bar = -0.064 on the Qwen3-8B trace).
//
// Input: the attention kernel's per-(row, kv tile) sums (sum P_hat, sum P).
// A tile is 128 query rows of one (batch, head) x one 128-key tile, and
//   epsilon_bar = mean over the tile's rows with sum P > 0 of (sum P_hat / sum P - 1),
// NaN when no row of the tile has mass (masked or never visited).
#include <cuda_runtime.h>
#include <math.h>

#include "hifa4_kernels.h"

namespace hifa4 {

// One thread per output tile; neighbouring threads take neighbouring kv
// tiles, so each row's sums are read as consecutive float2.
__global__ void __launch_bounds__(256) tile_stats_kernel(const float2* __restrict__ sums, long long n_out, int Nq,
                                                         int T, int nqa, float* __restrict__ eps_bar) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_out) return;
    const int t = (int)(idx % T);
    const int a = (int)((idx / T) % nqa);
    const long long bh = idx / ((long long)T * nqa);
    const int i0 = 128 * a, i1 = min(128 * a + 128, Nq);
    float acc = 0.0f;
    int cnt = 0;
    const float2* row0 = sums + ((size_t)bh * Nq) * T + t;
    // rows in order; eight loads in flight
    for (int i = i0; i < i1; i += 8) {
        float2 s[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) s[u] = i + u < i1 ? row0[(size_t)(i + u) * T] : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (s[u].y > 0.0f) {
                acc = __fadd_rn(acc, __fsub_rn(__fdiv_rn(s[u].x, s[u].y), 1.0f));
                ++cnt;
            }
        }
    }
    eps_bar[idx] = cnt > 0 ? __fdiv_rn(acc, (float)cnt) : __int_as_float(0x7FC00000);
}

cudaError_t launch_tile_stats(const float2* sums, int BH, int Nq, int T, float* eps_bar, cudaStream_t st) {
    const int nqa = (Nq + 127) / 128;
    const long long n = (long long)BH * nqa * T;
    if (n == 0) return cudaSuccess;
    const long long blocks = (n + 255) / 256;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    tile_stats_kernel<<<(unsigned)blocks, 256, 0, st>>>(sums, n, Nq, T, nqa, eps_bar);
    return cudaGetLastError();
}

}  // namespace hifa4
