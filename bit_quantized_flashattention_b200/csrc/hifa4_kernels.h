// Launchers shared between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hifa4 {

// One pass over Q (optional), K and V: smooth, quantize, write codes and
// MMA-ready scales.
struct QuantArgs {
    bool bf16;
    int D, G, hkv, nq, nkv, tiles_q;
    long long n_groups;           // B * Hkv
    const void* q;                // null: K and V only
    const void* k;
    const void* v;
    const float* s;
    const float* s_inv;
    uint8_t *qc, *qs, *kc, *ks, *vtc, *vts;
};

cudaError_t launch_quantize_qkv(const QuantArgs& a, cudaStream_t st);

cudaError_t launch_calibrate(bool bf16, const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, float alpha,
                             float* s, float* s_inv, cudaStream_t st);

struct AttnParams {
    const uint8_t* qs;       // MMA-ready scales of Q
    const uint8_t* ks;       // ... of K
    const uint8_t* vts;      // ... of V^T
    void* o;                 // [B,Hq,Nq,D] output
    float* lse;              // [B,Hq,Nq] or null
    uint8_t* p_codes;        // P_hat dump (debug variant only)
    uint8_t* p_sf;
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
// out_dtype 0 = f16, 1 = bf16, 2 = f32; dec: split-kv decode mode (D <= 128,
// G*Nq <= 64, at least 4 kv tiles; one CTA per group).
cudaError_t launch_attention(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const AttnParams& p, int D, int norm, bool causal, int out_dtype, bool dump, bool dec,
                             cudaStream_t st);

// Number of contiguous kv ranges the decode mode cuts the keys into.
constexpr int kDecodeSplits = 4;

}  // namespace hifa4
