// Smooth-QK calibration and 4-bit quantization kernels (sm_100a).
//
// HiFA4 abstract: Smooth-QK rescales Q by s and K by 1/s per channel, after
// RoPE and before quantization, with calibration-static factors; QK^T and PV
// then run as 4-bit GEMMs. Format: E2M1 elements, one E4M3 scale per 16
// elements along the contraction dimension (D for Q and K, tokens for V),
// round-to-nearest-even. Block rule:
//   sf = E4M3_rn_satfinite(amax * RN(1/6)),  r = RN(1/decode(sf)) (0 if sf = 0),
//   code = E2M1_rn_satfinite(RN(x * r)).
// These passes are HBM-bound streams: 128-bit loads and stores, one thread per
// 64 contiguous elements (four scale blocks = one 32-bit scale word in the
// MMA-ready scale layout, see hifa4.h).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hifa4_device.cuh"
#include "hifa4_kernels.h"

namespace hifa4 {

// Set (to the timeout status) when a bounded wait of the row pass expires;
// read and cleared by take_quantize_status.
__device__ uint32_t g_quantize_status;

cudaError_t take_quantize_status(uint32_t* out) {
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&word, g_quantize_status, sizeof(word));
    if (e == cudaSuccess && word != 0) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(g_quantize_status, &zero, sizeof(zero));
    }
    *out = word;
    return e;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Unpack 8 storage elements held in a 128-bit word.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
    const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = to_f32<T>(e[i]);
}

// Byte offset of (row r, scale k) inside a 512-byte scale atom.
__device__ __forceinline__ uint32_t atom_offset(uint32_t r) { return 16u * (r & 31u) + 4u * ((r >> 5) & 3u); }

// Reciprocal table RN(1/decode(sf)) for the 128 non-negative E4M3 codes
// (entry 0 = 0: a zero scale zeroes the block), built per CTA.
__device__ __forceinline__ void build_rcp_lut(float* lut) {
    for (unsigned i = threadIdx.x; i < 128; i += blockDim.x) lut[i] = (i == 0) ? 0.0f : __frcp_rn(e4m3_to_f32(i));
    __syncthreads();
}


// ------------------------------------------------- before quantization

// RoPE tables of one 8-channel chunk: cos and sin of the chunk's channel pairs
// at the row's position (clamped to the table).
struct RopeChunk {
    float4 c0, c1, s0, s1;
};

template <int D>
__device__ __forceinline__ RopeChunk load_rope(const float* cos_t, const float* sin_t, const int* pos, unsigned tok,
                                               int n_pos, unsigned chunk) {
    constexpr unsigned HALF = D / 16;                     // chunks per half row
    int ps = __ldg(pos + tok);
    ps = ps < 0 ? 0 : (ps >= n_pos ? n_pos - 1 : ps);
    const size_t off = (size_t)ps * (D / 2) + (chunk % HALF) * 8;
    const float4* c4 = reinterpret_cast<const float4*>(cos_t + off);
    const float4* s4 = reinterpret_cast<const float4*>(sin_t + off);
    return RopeChunk{__ldg(c4), __ldg(c4 + 1), __ldg(s4), __ldg(s4 + 1)};
}

// The rotation of one 8-channel chunk, rotate-half pairing: channel d < D/2
// pairs with d + D/2, which sits in chunk c ^ (D/16) of the same row, held by
// the lane LANE_XOR away (D/16 when a lane holds one chunk of the row, D/32
// when it holds two). Each product and sum is
// rounded on its own (no fused multiply-add):
//   first half   x <- RN(RN(x*cos) - RN(x_pair*sin))
//   second half  x <- RN(RN(x*cos) + RN(x_pair*sin))
// Every lane of the warp calls this (it shuffles).
template <typename T, int D, unsigned LANE_XOR = D / 16>
__device__ __forceinline__ void rope_chunk(const uint4& raw, unsigned chunk, const RopeChunk& t, float (&v)[8]) {
    constexpr unsigned HALF = D / 16;
    uint4 pr;
    pr.x = __shfl_xor_sync(0xFFFFFFFFu, raw.x, LANE_XOR);
    pr.y = __shfl_xor_sync(0xFFFFFFFFu, raw.y, LANE_XOR);
    pr.z = __shfl_xor_sync(0xFFFFFFFFu, raw.z, LANE_XOR);
    pr.w = __shfl_xor_sync(0xFFFFFFFFu, raw.w, LANE_XOR);
    float w[8];
    unpack8<T>(pr, w);
    const float cs[8] = {t.c0.x, t.c0.y, t.c0.z, t.c0.w, t.c1.x, t.c1.y, t.c1.z, t.c1.w};
    const float sn[8] = {t.s0.x, t.s0.y, t.s0.z, t.s0.w, t.s1.x, t.s1.y, t.s1.z, t.s1.w};
    if (chunk < HALF) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fsub_rn(__fmul_rn(v[i], cs[i]), __fmul_rn(w[i], sn[i]));
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fadd_rn(__fmul_rn(v[i], cs[i]), __fmul_rn(w[i], sn[i]));
    }
}

__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// ---------------------------------------------------------------- Q and K

// One row-quantization job (Q or K, quantized along D). A group holds the rows
// that share a kv head: for Q the G*Nq rows of its q heads stacked head after
// head (row p = head_in_group * n_tok + token), padded to whole 128-row tiles
// whose padding rows only receive zero scale words; for K the group's tokens.
// K rows may land at an offset of a larger output (a KV-cache append).
struct RowJob {
    const void* x;
    const float* scale;       // smoothing factors [Hkv, D] or null
    const float* rope_cos;    // RoPE tables [n_pos, D/2] (used by the RoPE variant)
    const float* rope_sin;
    const int* pos;           // position of each input token [n_tok]
    int n_pos;
    const float* mean;        // Q-Mean: subtract row (group*G + head_in_group) of [B*Hq, D], or null
    const float* bias_mean;   // Q-Mean on K rows: means [B*Hq, D] the score bias is taken from, or null
    float* bias;              // [B*Hq, rows_out] score bias output (with bias_mean)
    uint8_t* codes;
    uint8_t* sfs;
    unsigned n_tok;           // tokens per head in the input
    unsigned rows_in;         // input rows per group
    unsigned rows_out;        // output rows per group
    unsigned row0;            // output row of input row 0
    unsigned tiles_out;       // 128-row scale tiles per group in the output
    unsigned padded;          // rows [0, padded) are visited; [rows_in, padded) get zero scale words
    unsigned hkv;
    unsigned G;               // q heads per kv head
    unsigned blocks_per_group;
};

struct VJob {
    const void* v;
    uint8_t* vtc;
    uint8_t* vts;
    int n_in;                 // input tokens per group
    int nkv;                  // output tokens per group
    int start;                // output token of input token 0 (a multiple of 16)
    unsigned half0;           // first 64-token half of the output the job touches
    unsigned warps_per_group;
};

// A CTA quantizes a contiguous range of at most 4 row steps of its group (at
// most 32 KB of input, contiguous in memory). One thread moves the range into
// shared memory at the start with bulk copies, one per row step, each
// completing its own mbarrier: the whole range is in flight at once, and the
// arithmetic on a step starts as soon as it lands. Each lane owns one whole
// 16-element scale block of a row (its maximum needs no shuffle) and keeps
// that block's 16 smoothing factors in registers; products are formed two at
// a time (packed fp32 multiplies, each lane rounded on its own). The 4 scale
// bytes of a 64-element K step sit in 4 neighbouring lanes and are gathered by
// two shuffles into one 32-bit word of the MMA-ready atom. Before
// quantization, in order: RoPE (ROPE variant), the smoothing multiply, the
// Q-Mean subtraction; on K rows with bias_mean the Q-Mean score bias mean . K'
// of every head of the group is reduced across the row's lanes from the same
// pre-quantization values.
constexpr unsigned kRowStages = 4;                    // row steps (copy chunks) per CTA
constexpr unsigned kRowStageBytes = 4u * 256u * 32u;  // 4 row steps x 256 lanes x 32 bytes

// Sixteen values times sixteen factors, two at a time: v[i] <- RN(v[i] * f[i]).
__device__ __forceinline__ void mul16(float (&v)[16], const float (&f)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) unpack2(fmul2(pack2(v[i], v[i + 1]), pack2(f[i], f[i + 1])), v[i], v[i + 1]);
}

// Maximum of |v| over 16 values (three-input maxima; the maximum is exact).
__device__ __forceinline__ float absmax16(const float (&v)[16]) {
    float a[6];
#pragma unroll
    for (int i = 0; i < 5; ++i) a[i] = fmax3f(fabsf(v[3 * i]), fabsf(v[3 * i + 1]), fabsf(v[3 * i + 2]));
    a[5] = fabsf(v[15]);
    return fmax3f(fmax3f(a[0], a[1], a[2]), fmax3f(a[3], a[4], a[5]), 0.0f);
}

// Quantize 16 elements held by one thread (the rule in the file header).
__device__ __forceinline__ uint32_t quant_block16_lut(float (&x)[16], const float* lut, uint32_t& lo, uint32_t& hi) {
    const uint32_t sf = cvt_e4m3(__fmul_rn(absmax16(x), rn_one_sixth()));
    const float r = lut[sf & 127u];
    const float rr[16] = {r, r, r, r, r, r, r, r, r, r, r, r, r, r, r, r};
    mul16(x, rr);
    lo = cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
    hi = cvt_e2m1x8(x[8], x[9], x[10], x[11], x[12], x[13], x[14], x[15]);
    return sf;
}

template <typename T, int D, bool ROPE, bool QM>
__device__ __forceinline__ void quantize_rows_cta(const RowJob& jb, unsigned cta, const float* lut, uint8_t* stage,
                                                  uint64_t* bars, unsigned long long limit_ns, bool stall) {
    constexpr unsigned CPR = D / 16;                       // lanes (scale blocks) per row
    constexpr unsigned RPB = 256 / CPR;                    // rows per CTA step
    constexpr unsigned ROW_BYTES = D * sizeof(T);
    constexpr unsigned KS = D / 64;
    const unsigned grp = cta / jb.blocks_per_group;
    const unsigned part = cta % jb.blocks_per_group;
    const unsigned c = threadIdx.x % CPR;                  // the lane's block of the row
    const unsigned steps = (jb.padded + RPB - 1) / RPB;
    const unsigned s0 = (unsigned)(((unsigned long long)steps * part) / jb.blocks_per_group);
    const unsigned s1 = (unsigned)(((unsigned long long)steps * (part + 1)) / jb.blocks_per_group);
    float sc[16];
    if (jb.scale != nullptr) {
        const float* sp = jb.scale + (size_t)(grp % jb.hkv) * D + c * 16;
        float a[8], b[8];
        load8(sp, a);
        load8(sp + 8, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) { sc[i] = a[i]; sc[8 + i] = b[i]; }
    }
    const T* xg = static_cast<const T*>(jb.x) + (size_t)grp * jb.rows_in * D;
    uint8_t* cg = jb.codes + ((size_t)grp * jb.rows_out + jb.row0) * (D / 2);
    uint8_t* sg = jb.sfs + (size_t)grp * jb.tiles_out * KS * 512;
    const unsigned r_in = threadIdx.x / CPR;
    const unsigned row_first = s0 * RPB;                   // first row of the range
    if (threadIdx.x == 0 && !stall) {
        for (unsigned k = 0; k < kRowStages; ++k) {
            const unsigned a = min(min(s0 + k, s1) * RPB, jb.rows_in);
            const unsigned b = min(min(s0 + k + 1, s1) * RPB, jb.rows_in);
            if (b > a) {
                mbar_arrive_expect_tx(&bars[k], (b - a) * ROW_BYTES);
                bulk_load(stage + (a - row_first) * ROW_BYTES, xg + (size_t)a * D, (b - a) * ROW_BYTES, &bars[k]);
            } else {
                mbar_arrive(&bars[k]);
            }
        }
    }
    for (unsigned st = s0, k = 0; st < s1; ++st, ++k) {
        // step k has landed (bounded: on expiry the status is recorded, the
        // remaining copies are drained and the CTA stops)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_drain(&bars[k], 0, limit_ns))) {
            if (threadIdx.x == 0) {
                atomicExch(&g_quantize_status, kStatusTimeout);
                if (!stall)
                    for (unsigned kk = k; kk < kRowStages; ++kk) mbar_wait_drain(&bars[kk], 0, limit_ns);
            }
            return;
        }
        const unsigned p = st * RPB + r_in;
        const bool real = p < jb.rows_in;
        uint4 raw0 = make_uint4(0u, 0u, 0u, 0u), raw1 = raw0;
        if (real) {
            const uint4* src = reinterpret_cast<const uint4*>(stage + (p - row_first) * ROW_BYTES + c * 32);
            raw0 = src[0];
            raw1 = src[1];
        }
        float v[16];
        {
            float a[8], b[8];
            unpack8<T>(raw0, a);
            unpack8<T>(raw1, b);
            if constexpr (ROPE) {
                // the table rows are cache hits: loaded where they are used
                const unsigned tok = real ? p % jb.n_tok : 0u;
                rope_chunk<T, D, D / 32>(raw0, 2 * c, load_rope<D>(jb.rope_cos, jb.rope_sin, jb.pos, tok, jb.n_pos, 2 * c), a);
                rope_chunk<T, D, D / 32>(raw1, 2 * c + 1,
                                         load_rope<D>(jb.rope_cos, jb.rope_sin, jb.pos, tok, jb.n_pos, 2 * c + 1), b);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) { v[i] = a[i]; v[8 + i] = b[i]; }
        }
        if (jb.scale != nullptr) mul16(v, sc);
        if (QM && jb.mean != nullptr && real) {
            const float* mp = jb.mean + ((size_t)grp * jb.G + p / jb.n_tok) * D + c * 16;
            float a[8], b[8];
            load8(mp, a);
            load8(mp + 8, b);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[i] = __fsub_rn(v[i], a[i]);
                v[8 + i] = __fsub_rn(v[8 + i], b[i]);
            }
        }
        if (QM && jb.bias_mean != nullptr) {
            // score bias of this key for every q head of the group
            for (unsigned hl = 0; hl < jb.G; ++hl) {
                float acc = 0.0f;
                if (real) {
                    const float* mp = jb.bias_mean + ((size_t)grp * jb.G + hl) * D + c * 16;
                    float a[8], b[8];
                    load8(mp, a);
                    load8(mp + 8, b);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = __fmaf_rn(a[i], v[i], acc);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = __fmaf_rn(b[i], v[8 + i], acc);
                }
#pragma unroll
                for (unsigned o = CPR / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
                if (real && c == 0) jb.bias[((size_t)grp * jb.G + hl) * jb.rows_out + jb.row0 + p] = acc;
            }
        }
        uint32_t lo, hi;
        const uint32_t sf = quant_block16_lut(v, lut, lo, hi);
        if (real) *reinterpret_cast<uint2*>(cg + (size_t)p * (D / 2) + c * 8) = make_uint2(lo, hi);
        uint32_t word = sf << (8u * (c & 3u));
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        const unsigned q = jb.row0 + p;                    // output row
        if (p < jb.padded && (c & 3u) == 0u)
            *reinterpret_cast<uint32_t*>(sg + ((size_t)(q >> 7) * KS + c / 4) * 512 + atom_offset(q & 127u)) =
                real ? word : 0u;
    }
}

// ---------------------------------------------------------------------- V

// V quantized along tokens, written transposed and tiled (each 128-token tile
// of V^T is one contiguous D x 64-byte block). A warp covers 32 channels x 64
// output tokens of one group; lane (cc, tb) owns 4 channels (cc = 0..7) x one
// 16-token block (tb = 0..3): it reads 16 rows of 8 bytes (each load
// instruction reads 4 rows of 64 contiguous bytes), quantizes one block per
// channel and writes 8 code bytes per channel. The 4 scale bytes of a channel
// for the 64-token half are gathered by shuffles into one word when the job
// covers the whole half; a job that covers part of it (an append) writes its
// blocks' scale bytes one by one and leaves the others alone. For D = 64 one
// warp per half also fills the padding rows of the scale atoms (row 64 = 1.0
// for the normalizer column of P-Reordering, the rest 0).
template <typename T, int D>
__device__ __forceinline__ void quantize_v_warp(const VJob& jb, unsigned gw_all, const float* lut) {
    constexpr int NRB = (D + 127) / 128;
    constexpr unsigned CWARPS = D / 32;                    // warps per 64-token half (32 channels each)
    const unsigned lane = threadIdx.x & 31u;
    const unsigned grp = gw_all / jb.warps_per_group;
    const unsigned gw = gw_all % jb.warps_per_group;
    const int nkv = jb.nkv;
    const unsigned cw = gw % CWARPS;
    const unsigned hh = jb.half0 + gw / CWARPS;            // 64-token half of the output
    const unsigned cc = lane >> 2, tb = lane & 3u;
    const unsigned d0 = cw * 32 + cc * 4;
    const int tok0 = (int)(hh * 64 + tb * 16);             // output token of this lane's block
    const bool active = tok0 >= jb.start && tok0 < jb.start + jb.n_in;
    const bool whole = (int)(hh * 64) >= jb.start && (int)(hh * 64 + 64) <= jb.start + jb.n_in;   // warp-uniform
    uint2 raw[16];
    if (active) {
        const T* src = static_cast<const T*>(jb.v) + ((size_t)grp * jb.n_in + (tok0 - jb.start)) * D + d0;
#pragma unroll
        for (int i = 0; i < 16; ++i) raw[i] = *reinterpret_cast<const uint2*>(src + (size_t)i * D);
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) raw[i] = make_uint2(0u, 0u);
    }
    const unsigned j = hh / 2, half = hh % 2;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = to_f32<T>(reinterpret_cast<const T*>(&raw[i])[k]);
        uint32_t lo, hi;
        const uint32_t sf = quant_block16_lut(x, lut, lo, hi);
        const unsigned d = d0 + k;
        // tiled V^T codes: the 64 bytes of channel d for kv tile tok0/128
        if (active)
            *reinterpret_cast<uint2*>(jb.vtc + (((size_t)grp * (nkv / 128) + tok0 / 128) * D + d) * 64 +
                                      (tok0 % 128) / 2) = make_uint2(lo, hi);
        const size_t atom = (((size_t)grp * (nkv / 128) + j) * NRB + (d >> 7)) * 2 + half;
        if (whole) {
            uint32_t word = sf << (8u * tb);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
            if (tb == 0) *reinterpret_cast<uint32_t*>(jb.vts + atom * 512 + atom_offset(d & 127u)) = word;
        } else if (active) {
            jb.vts[atom * 512 + atom_offset(d & 127u) + tb] = (uint8_t)sf;
        }
    }
    if constexpr (D == 64) {
        if (cw == 0) {
            const size_t atom = ((size_t)grp * (nkv / 128) + j) * 2 + half;
            for (unsigned r = 64 + lane; r < 128; r += 32)
                *reinterpret_cast<uint32_t*>(jb.vts + atom * 512 + atom_offset(r)) = (r == 64) ? 0x38383838u : 0u;
        }
    }
}

// One launch for the whole pass: CTAs [0, nq) quantize Q rows, [nq, nq + nk)
// K rows, the rest V (8 warps per CTA).
template <typename T, int D, bool ROPE, bool QM>
__global__ void __launch_bounds__(256) quantize_qkv_kernel(RowJob q, RowJob k, VJob v, unsigned nq, unsigned nk,
                                                           unsigned v_warps, unsigned long long limit_ns, int stall) {
    __shared__ float lut[128];
    __shared__ uint64_t bars[kRowStages];
    extern __shared__ __align__(128) uint8_t stage[];      // kRowStageBytes (row CTAs)
    // the next kernel (attention) may be scheduled as these CTAs retire; it
    // waits for this grid's completion before reading the packed operands
    launch_dependents();
    const unsigned b = blockIdx.x;
    if (threadIdx.x == 0 && b < nq + nk) {
        for (unsigned i = 0; i < kRowStages; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
    }
    build_rcp_lut(lut);                                    // ends with a CTA barrier
    if (b < nq) {
        quantize_rows_cta<T, D, ROPE, QM>(q, b, lut, stage, bars, limit_ns, stall != 0);
    } else if (b < nq + nk) {
        quantize_rows_cta<T, D, ROPE, QM>(k, b - nq, lut, stage, bars, limit_ns, stall != 0);
    } else {
        const unsigned gw = (b - nq - nk) * 8 + (threadIdx.x >> 5);
        if (gw < v_warps) quantize_v_warp<T, D>(v, gw, lut);
    }
}

// ----------------------------------------------------------------- Q-Mean

// Per-(batch, head, channel) mean of the pre-quantization Q (after RoPE and
// smoothing) over the head's Nq tokens: the sum is accumulated in fp64, then
// divided in fp64 and rounded once to fp32. A thread-block cluster of CL CTAs
// serves one (b, h): CTA rank r sums the tokens [r*Nq/CL, (r+1)*Nq/CL) (lane
// chunk c = tid % (D/8) of token lane tid / (D/8)), reduces its token lanes
// through shared memory in a fixed order, and rank 0 adds the CL partial sums
// from the other CTAs' shared memory (distributed shared memory), in rank order.
struct QMeanJob {
    const void* q;
    const float* scale;       // smoothing factors [Hkv, D] or null
    const float* rope_cos;
    const float* rope_sin;
    const int* pos;
    int n_pos;
    float* mean;              // [B*Hq, D]
    int Hq, G, Hkv, Nq;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// fp64 load from the shared memory of CTA `rank` of this cluster
__device__ __forceinline__ double ld_cluster_f64(const double* local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(remote) : "memory");
    return v;
}

template <typename T, int D, bool ROPE>
__global__ void __launch_bounds__(256) q_mean_kernel(QMeanJob jb) {
    constexpr unsigned CPR = D / 8, TL = 256 / CPR;
    __shared__ double red[TL][D];
    __shared__ double part[D];
    const unsigned cl = cluster_size(), rank = cluster_rank();
    const unsigned bh = blockIdx.x / cl;
    const unsigned c = threadIdx.x % CPR, tl = threadIdx.x / CPR;
    const unsigned g = (bh % (unsigned)jb.Hq) / (unsigned)jb.G;
    float sc[8];
    if (jb.scale != nullptr) load8(jb.scale + (size_t)g * D + c * 8, sc);
    const unsigned t_begin = (unsigned)(((unsigned long long)jb.Nq * rank) / cl);
    const unsigned t_end = (unsigned)(((unsigned long long)jb.Nq * (rank + 1)) / cl);
    const T* xb = static_cast<const T*>(jb.q) + (size_t)bh * jb.Nq * D;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    for (unsigned base = t_begin; base < t_end; base += TL) {        // warp-uniform trip count
        const unsigned i = base + tl;
        const bool real = i < t_end;
        const uint4 raw = real ? *reinterpret_cast<const uint4*>(xb + (size_t)i * D + c * 8) : make_uint4(0u, 0u, 0u, 0u);
        float v[8];
        unpack8<T>(raw, v);
        if constexpr (ROPE) {
            const RopeChunk rc = load_rope<D>(jb.rope_cos, jb.rope_sin, jb.pos, real ? i : 0u, jb.n_pos, c);
            rope_chunk<T, D>(raw, c, rc, v);
        }
        if (jb.scale != nullptr) {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], sc[e]);
        }
        if (real) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __dadd_rn(acc[e], (double)v[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[tl][c * 8 + e] = acc[e];
    __syncthreads();
    for (unsigned d = threadIdx.x; d < (unsigned)D; d += 256) {
        double sum = 0.0;
        for (unsigned t = 0; t < TL; ++t) sum = __dadd_rn(sum, red[t][d]);
        part[d] = sum;
    }
    cluster_sync_all();                       // every CTA's partial sums are in its shared memory
    if (rank == 0) {
        for (unsigned d = threadIdx.x; d < (unsigned)D; d += 256) {
            double sum = part[d];
            for (unsigned r = 1; r < cl; ++r) sum = __dadd_rn(sum, ld_cluster_f64(&part[d], r));
            jb.mean[(size_t)bh * D + d] = __double2float_rn(__ddiv_rn(sum, (double)jb.Nq));
        }
    }
    cluster_sync_all();                       // rank 0 has read the others' shared memory
}

// ------------------------------------------------------------ calibration

// Per (kv head, channel) maxima of |Q| (over the group's q heads) and |K|,
// accumulated with atomicMax on the bit patterns of non-negative floats into
// aq_bits / ak_bits (zeroed beforehand). One CTA per (slice, 64-token chunk),
// one thread per channel.
template <typename T>
__global__ void calib_amax_kernel(const T* __restrict__ x, int heads, int n, int d, int heads_per_kv, int hkv,
                                  uint32_t* __restrict__ amax_bits) {
    const long long slice = blockIdx.y;                 // b * heads + h
    const int h = (int)(slice % heads);
    const int g = (h / heads_per_kv) % hkv;
    const int t0 = blockIdx.x * 64;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float m = 0.0f;
        const T* p = x + ((size_t)slice * n + t0) * d + c;
        const int tn = min(64, n - t0);
        for (int t = 0; t < tn; ++t) m = fmaxf(m, fabsf(to_f32<T>(p[(size_t)t * d])));
        atomicMax(amax_bits + (size_t)g * d + c, __float_as_uint(m));
    }
}

__global__ void calib_finalize_kernel(float* __restrict__ s, float* __restrict__ s_inv, int count, float alpha) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    const float aq = __uint_as_float(reinterpret_cast<const uint32_t*>(s)[i]);
    const float ak = __uint_as_float(reinterpret_cast<const uint32_t*>(s_inv)[i]);
    float sv;
    if (aq == 0.0f || ak == 0.0f) {
        sv = 1.0f;
    } else if (alpha == 0.5f) {
        sv = __fsqrt_rn(__fdiv_rn(ak, aq));
    } else {
        sv = (float)(pow((double)ak, (double)alpha) / pow((double)aq, 1.0 - (double)alpha));
    }
    s[i] = sv;
    s_inv[i] = __frcp_rn(sv);
}

// ------------------------------------------------------------ launchers

template <typename T, int D>
static cudaError_t launch_qkv_t(const QuantArgs& a, cudaStream_t st) {
    const long long n_grp = a.n_groups;
    // small CTAs (at most kRowStages row steps of 256/(D/16) rows each): many
    // CTAs per SM overlap one CTA's loads with another's arithmetic
    const long long rows_per_step = 256 / (D / 16);
    auto per_group = [&](long long padded_rows) -> long long {
        if (padded_rows == 0) return 0;
        const long long steps = (padded_rows + rows_per_step - 1) / rows_per_step;
        return (steps + kRowStages - 1) / kRowStages;
    };
    const bool rope = a.rope_cos != nullptr;
    RowJob jq{};
    jq.x = a.q;
    jq.scale = a.s;
    jq.rope_cos = a.rope_cos;
    jq.rope_sin = a.rope_sin;
    jq.pos = a.q_pos;
    jq.n_pos = a.n_pos;
    jq.mean = a.q_mean;
    jq.codes = a.qc;
    jq.sfs = a.qs;
    jq.n_tok = (unsigned)a.nq;
    jq.rows_in = jq.rows_out = (unsigned)(a.G * a.nq);
    jq.tiles_out = (unsigned)a.tiles_q;
    jq.padded = (unsigned)a.tiles_q * 128u;
    jq.hkv = (unsigned)a.hkv;
    jq.G = (unsigned)a.G;
    jq.blocks_per_group = (unsigned)per_group(a.q != nullptr ? jq.padded : 0);
    RowJob jk{};
    jk.x = a.k;
    jk.scale = a.s_inv;
    jk.rope_cos = a.rope_cos;
    jk.rope_sin = a.rope_sin;
    jk.pos = a.k_pos;
    jk.n_pos = a.n_pos;
    jk.bias_mean = a.q_mean;
    jk.bias = a.s_bias;
    jk.codes = a.kc;
    jk.sfs = a.ks;
    jk.n_tok = jk.rows_in = jk.padded = (unsigned)a.nkv_in;
    jk.rows_out = (unsigned)a.nkv;
    jk.row0 = (unsigned)a.kv_start;
    jk.tiles_out = (unsigned)(a.nkv / 128);
    jk.hkv = (unsigned)a.hkv;
    jk.G = (unsigned)a.G;
    jk.blocks_per_group = (unsigned)per_group(jk.padded);
    VJob jv{};
    jv.v = a.v;
    jv.vtc = a.vtc;
    jv.vts = a.vts;
    jv.n_in = a.nkv_in;
    jv.nkv = a.nkv;
    jv.start = a.kv_start;
    jv.half0 = (unsigned)(a.kv_start / 64);
    const unsigned halves =
        a.nkv_in > 0 ? (unsigned)((a.kv_start + a.nkv_in - 1) / 64 - a.kv_start / 64 + 1) : 0u;   // 0: Q only
    jv.warps_per_group = halves * (D / 32);
    const long long v_warps = n_grp * jv.warps_per_group;
    const long long v_ctas = (v_warps + 7) / 8;
    const long long nq = a.q != nullptr ? n_grp * jq.blocks_per_group : 0;
    const long long nk = n_grp * jk.blocks_per_group;
    const long long total = nq + nk + v_ctas;
    if (total > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    // variants: RoPE or not, Q-Mean or not (the plain pass carries neither)
    const bool qm = a.q_mean != nullptr;
    auto kern = rope ? (qm ? quantize_qkv_kernel<T, D, true, true> : quantize_qkv_kernel<T, D, true, false>)
                     : (qm ? quantize_qkv_kernel<T, D, false, true> : quantize_qkv_kernel<T, D, false, false>);
    const int smem = (nq + nk > 0) ? (int)kRowStageBytes : 0;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRowStageBytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)total, 256, smem, st>>>(jq, jk, jv, (unsigned)nq, (unsigned)nk, (unsigned)v_warps,
                                              a.wait_limit_ns, a.stall_loads);
    return cudaGetLastError();
}

cudaError_t launch_quantize_qkv(const QuantArgs& a, cudaStream_t st) {
    switch (a.D) {
        case 64: return a.bf16 ? launch_qkv_t<__nv_bfloat16, 64>(a, st) : launch_qkv_t<__half, 64>(a, st);
        case 128: return a.bf16 ? launch_qkv_t<__nv_bfloat16, 128>(a, st) : launch_qkv_t<__half, 128>(a, st);
        case 256: return a.bf16 ? launch_qkv_t<__nv_bfloat16, 256>(a, st) : launch_qkv_t<__half, 256>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int D>
static cudaError_t launch_q_mean_t(const QMeanArgs& a, cudaStream_t st) {
    QMeanJob jb{a.q, a.s, a.rope_cos, a.rope_sin, a.q_pos, a.n_pos, a.mean, a.Hq, a.Hq / a.Hkv, a.Hkv, a.Nq};
    // one cluster per (b, h); more CTAs per cluster for long heads (at least
    // 256 tokens each), at most the portable cluster size of 8
    unsigned cl = 1;
    while (cl < 8 && (long long)a.Nq >= 256LL * cl * 2) cl *= 2;
    const long long n = (long long)a.B * a.Hq * cl;
    if (n > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3((unsigned)n);
    lc.blockDim = dim3(256);
    lc.dynamicSmemBytes = 0;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    if (a.rope_cos != nullptr) return cudaLaunchKernelEx(&lc, q_mean_kernel<T, D, true>, jb);
    return cudaLaunchKernelEx(&lc, q_mean_kernel<T, D, false>, jb);
}

cudaError_t launch_q_mean(const QMeanArgs& a, cudaStream_t st) {
    switch (a.D) {
        case 64: return a.bf16 ? launch_q_mean_t<__nv_bfloat16, 64>(a, st) : launch_q_mean_t<__half, 64>(a, st);
        case 128: return a.bf16 ? launch_q_mean_t<__nv_bfloat16, 128>(a, st) : launch_q_mean_t<__half, 128>(a, st);
        case 256: return a.bf16 ? launch_q_mean_t<__nv_bfloat16, 256>(a, st) : launch_q_mean_t<__half, 256>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
static cudaError_t launch_calib_t(const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, float alpha,
                                  float* s, float* s_inv, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(s, 0, sizeof(float) * (size_t)Hkv * D, st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(s_inv, 0, sizeof(float) * (size_t)Hkv * D, st);
    if (e != cudaSuccess) return e;
    const int threads = D < 256 ? D : 256;
    const unsigned chunks = (unsigned)((N + 63) / 64);
    if ((long long)B * Hq > 65535) return cudaErrorInvalidConfiguration;
    calib_amax_kernel<T><<<dim3(chunks, (unsigned)(B * Hq)), threads, 0, st>>>(
        static_cast<const T*>(q), Hq, N, D, Hq / Hkv, Hkv, reinterpret_cast<uint32_t*>(s));
    calib_amax_kernel<T><<<dim3(chunks, (unsigned)(B * Hkv)), threads, 0, st>>>(
        static_cast<const T*>(k), Hkv, N, D, 1, Hkv, reinterpret_cast<uint32_t*>(s_inv));
    const int count = Hkv * D;
    calib_finalize_kernel<<<(count + 255) / 256, 256, 0, st>>>(s, s_inv, count, alpha);
    return cudaGetLastError();
}

cudaError_t launch_calibrate(bool bf16, const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, float alpha,
                             float* s, float* s_inv, cudaStream_t st) {
    if (bf16) return launch_calib_t<__nv_bfloat16>(q, k, B, Hq, Hkv, N, D, alpha, s, s_inv, st);
    return launch_calib_t<__half>(q, k, B, Hq, Hkv, N, D, alpha, s, s_inv, st);
}

}  // namespace hifa4
