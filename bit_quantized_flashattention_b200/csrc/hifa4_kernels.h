// Launchers shared between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hifa4 {

// One pass over Q (optional), K and V: quantize, write codes and MMA-ready
// scales. Before quantization, in order: RoPE (rope_cos non-null), the Smooth-QK
// multiply (s / s_inv non-null), the Q-Mean subtraction on Q (q_mean
// non-null; the K pass then writes the score bias s_bias). The K and V input
// tokens [0, nkv_in) land at tokens [kv_start, kv_start + nkv_in) of an output
// of nkv tokens (a KV-cache append; the plain pass has nkv_in = nkv, kv_start = 0;
// nkv_in = 0 quantizes Q alone).
struct QuantArgs {
    bool bf16;
    int D, G, hkv, nq, nkv, tiles_q;
    int nkv_in, kv_start;
    long long n_groups;           // B * Hkv
    const void* q;                // null: K and V only
    const void* k;
    const void* v;
    const float* s;
    const float* s_inv;
    const float* rope_cos;        // [n_pos, D/2] or null
    const float* rope_sin;
    const int* q_pos;             // [nq]
    const int* k_pos;             // [nkv_in]
    int n_pos;
    const float* q_mean;          // [B*Hq, D] or null
    float* s_bias;                // [B*Hq, nkv]
    uint8_t *qc, *qs, *kc, *ks, *vtc, *vts;
    unsigned long long wait_limit_ns;   // bound of the copy waits of the row pass
    int stall_loads;                    // test hook: the row pass issues no copies (its waits time out)
};

cudaError_t launch_quantize_qkv(const QuantArgs& a, cudaStream_t st);

// Synchronous: the quantize pass's status word (0, or HIFA4_ERR_TIMEOUT when
// a bounded wait expired in it since the last call), then clears it.
cudaError_t take_quantize_status(uint32_t* out);

// Q-Mean: mean [B*Hq, D] of the pre-quantization Q (RoPE, smoothing as above).
struct QMeanArgs {
    bool bf16;
    int B, Hq, Hkv, Nq, D;
    const void* q;
    const float* s;
    const float* rope_cos;
    const float* rope_sin;
    const int* q_pos;
    int n_pos;
    float* mean;
};

cudaError_t launch_q_mean(const QMeanArgs& a, cudaStream_t st);

cudaError_t launch_calibrate(bool bf16, const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, float alpha,
                             float* s, float* s_inv, cudaStream_t st);

struct AttnParams {
    const uint8_t* qs;       // MMA-ready scales of Q
    const uint8_t* ks;       // ... of K
    const uint8_t* vts;      // ... of V^T
    void* o;                 // [B,Hq,Nq,D] output
    float* lse;              // [B,Hq,Nq] or null
    // optional outputs and inputs of the extras variant (each may be null)
    const float* s_bias;     // [B*Hq, Nkv] added to the scores of head (b, h)
    uint8_t* p_codes;        // P_hat dump [B*Hq*Nq, Nkv/2]
    uint8_t* p_sf;           // ... and its scales [B*Hq*Nq, Nkv/16]
    float2* tile_sums;       // (sum P_hat, sum P) per (row, kv tile) [B*Hq*Nq, Nkv/128]
    // in-kernel Q quantization (variant 3; Q itself comes through the Q tensor map)
    const float* q_scale;    // Smooth-QK factors [Hkv, D] or null
    int q_bf16;
    uint32_t* status;        // workspace status word
    int B, Hq, Hkv, Nq, Nkv, G;
    int Tq;                  // 128-row tiles per (b, kv head) group
    int n_kv_tiles;          // Nkv / 128
    int n_work;              // grid size (work units)
    int heavy_first;         // causal: longest tiles first
    float c;                 // RN(sm_scale * log2 e)
    unsigned long long wait_limit_ns;
    int stall_loads;         // test hook: issue no loads (all waits time out)
};

// D in {64,128,256}; norm 0 = P-Reordering, 1 = high-precision l;
// out_dtype 0 = f16, 1 = bf16, 2 = f32; xt: 0 the plain variant, 1 adds
// s_bias, 2 also writes p_codes / p_sf / tile_sums where they are non-null,
// 3 quantizes Q itself, reading the caller's Q through tmQ (D = 128, not dec); dec: split-kv decode mode (D <= 128,
// G*Nq <= 64, at least 4 kv tiles; one CTA per group).
cudaError_t launch_attention(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const AttnParams& p, int D, int norm, bool causal, int out_dtype, int xt, bool dec,
                             cudaStream_t st);

// Per-tile epsilon-bar from the attention kernel's tile sums.
cudaError_t launch_tile_stats(const float2* sums, int BH, int Nq, int T, float* eps_bar, cudaStream_t st);

// Number of contiguous kv ranges the decode mode cuts the keys into.
constexpr int kDecodeSplits = 4;

}  // namespace hifa4
