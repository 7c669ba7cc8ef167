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

// Quantize 16 elements held by one thread (the rule in the file header).
__device__ __forceinline__ uint32_t quant_block16_lut(const float (&x)[16], const float* lut, uint32_t& lo,
                                                      uint32_t& hi) {
    float amax = fabsf(x[0]);
#pragma unroll
    for (int i = 1; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint32_t sf = cvt_e4m3(__fmul_rn(amax, rn_one_sixth()));
    const float r = lut[sf & 127u];
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(x[i], r);
    lo = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    hi = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
    return sf;
}

// ---------------------------------------------------------------- Q and K

// One row-quantization job (Q or K, quantized along D). A group is the G*N
// consecutive input rows that share a kv head (G = q heads per kv head for Q,
// 1 for K), padded to whole 128-row tiles; padding rows only receive zero
// scale words.
struct RowJob {
    const void* x;
    const float* scale;       // smoothing factors [Hkv, D] or null
    uint8_t* codes;
    uint8_t* sfs;
    unsigned rows_per_group;
    unsigned tiles_per_group;
    unsigned hkv;
    unsigned blocks_per_group;  // CTAs sharing one group's rows
};

struct VJob {
    const void* v;
    uint8_t* vtc;
    uint8_t* vts;
    int nkv;
    unsigned warps_per_group;
};

// Each lane owns one 8-element chunk of a row (a warp instruction reads 512
// contiguous bytes); a CTA walks a contiguous range of its group's rows, four
// row steps per iteration so that four loads per lane are in flight. The
// lane's 8 smoothing factors stay in registers. The two halves of a
// 16-element block sit in neighbouring lanes (one shuffle for the maximum),
// and the 4 scale bytes of a 64-element K step are gathered by shuffles into
// one 32-bit word of the MMA-ready atom.
template <typename T, int D>
__device__ __forceinline__ void quantize_rows_cta(const RowJob& jb, unsigned cta, const float* lut) {
    constexpr unsigned CPR = D / 8;                        // chunks per row
    constexpr unsigned RPB = 256 / CPR;                    // rows per CTA step
    constexpr unsigned UNROLL = 4;
    constexpr unsigned KS = D / 64;
    const unsigned grp = cta / jb.blocks_per_group;
    const unsigned part = cta % jb.blocks_per_group;
    const unsigned c = threadIdx.x % CPR;
    const unsigned padded = jb.tiles_per_group * 128;
    const unsigned steps = (padded + RPB - 1) / RPB;
    const unsigned s0 = (unsigned)(((unsigned long long)steps * part) / jb.blocks_per_group);
    const unsigned s1 = (unsigned)(((unsigned long long)steps * (part + 1)) / jb.blocks_per_group);
    float sc[8];
    if (jb.scale != nullptr) {
        const float4* s4 = reinterpret_cast<const float4*>(jb.scale + (size_t)(grp % jb.hkv) * D + c * 8);
        const float4 a = __ldg(s4), b = __ldg(s4 + 1);
        sc[0] = a.x; sc[1] = a.y; sc[2] = a.z; sc[3] = a.w;
        sc[4] = b.x; sc[5] = b.y; sc[6] = b.z; sc[7] = b.w;
    }
    const T* xg = static_cast<const T*>(jb.x) + (size_t)grp * jb.rows_per_group * D;
    uint8_t* cg = jb.codes + (size_t)grp * jb.rows_per_group * (D / 2);
    uint8_t* sg = jb.sfs + (size_t)grp * jb.tiles_per_group * KS * 512;
    const unsigned r_in = threadIdx.x / CPR;
    for (unsigned st = s0; st < s1; st += UNROLL) {
        uint4 raw[UNROLL];
#pragma unroll
        for (unsigned u = 0; u < UNROLL; ++u) {
            const unsigned pp = (st + u) * RPB + r_in;
            raw[u] = (st + u < s1 && pp < jb.rows_per_group)
                         ? *reinterpret_cast<const uint4*>(xg + (size_t)pp * D + c * 8)
                         : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (unsigned u = 0; u < UNROLL; ++u) {
            const unsigned p = (st + u) * RPB + r_in;
            const bool in_range = st + u < s1;             // warp-uniform
            const bool real = in_range && p < jb.rows_per_group;
            float v[8];
            unpack8<T>(raw[u], v);
            if (jb.scale != nullptr) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], sc[i]);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
            const uint32_t sf = cvt_e4m3(__fmul_rn(amax, rn_one_sixth()));
            const float r = lut[sf & 127u];
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(v[i], r);
            const uint32_t w = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
            if (real) *reinterpret_cast<uint32_t*>(cg + (size_t)p * (D / 2) + c * 4) = w;
            uint32_t word = ((c & 1u) == 0u) ? (sf << (8u * ((c >> 1) & 3u))) : 0u;
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
            if (in_range && p < padded && (c & 7u) == 0u)
                *reinterpret_cast<uint32_t*>(sg + ((size_t)(p >> 7) * KS + c / 8) * 512 + atom_offset(p & 127u)) =
                    real ? word : 0u;
        }
    }
}

// ---------------------------------------------------------------------- V

// V quantized along tokens, written transposed and tiled (each 128-token tile
// of V^T is one contiguous D x 64-byte block). A warp covers 32 channels x 64
// tokens of one group; lane (cc, tb) owns 4 channels (cc = 0..7) x one 16-token
// block (tb = 0..3): it reads 16 rows of 8 bytes (each load instruction reads 4
// rows of 64 contiguous bytes), quantizes one block per channel and writes 8
// code bytes per channel; the 4 scale bytes of a channel for the 64-token half
// come from the lanes tb = 0..3 and are gathered by shuffles. For D = 64 one
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
    const unsigned hh = gw / CWARPS;                       // 64-token half over the sequence
    const unsigned cc = lane >> 2, tb = lane & 3u;
    const unsigned d0 = cw * 32 + cc * 4;
    const unsigned tok0 = hh * 64 + tb * 16;
    const T* src = static_cast<const T*>(jb.v) + ((size_t)grp * nkv + tok0) * D + d0;
    uint2 raw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) raw[i] = *reinterpret_cast<const uint2*>(src + (size_t)i * D);
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
        *reinterpret_cast<uint2*>(jb.vtc + (((size_t)grp * (nkv / 128) + tok0 / 128) * D + d) * 64 + (tok0 % 128) / 2) =
            make_uint2(lo, hi);
        uint32_t word = sf << (8u * tb);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        if (tb == 0) {
            const size_t atom = (((size_t)grp * (nkv / 128) + j) * NRB + (d >> 7)) * 2 + half;
            *reinterpret_cast<uint32_t*>(jb.vts + atom * 512 + atom_offset(d & 127u)) = word;
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
template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_qkv_kernel(RowJob q, RowJob k, VJob v, unsigned nq, unsigned nk,
                                                           unsigned v_warps) {
    __shared__ float lut[128];
    // the next kernel (attention) may be scheduled as these CTAs retire; it
    // waits for this grid's completion before reading the packed operands
    launch_dependents();
    build_rcp_lut(lut);
    const unsigned b = blockIdx.x;
    if (b < nq) {
        quantize_rows_cta<T, D>(q, b, lut);
    } else if (b < nq + nk) {
        quantize_rows_cta<T, D>(k, b - nq, lut);
    } else {
        const unsigned gw = (b - nq - nk) * 8 + (threadIdx.x >> 5);
        if (gw < v_warps) quantize_v_warp<T, D>(v, gw, lut);
    }
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
    int dev = 0, sms = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_qkv_kernel<T, D>, 256, 0) != cudaSuccess || occ < 1)
        occ = 1;
    (void)occ;
    (void)sms;
    const long long n_grp = a.n_groups;
    // small CTAs (at most 8 row steps of 256/(D/8) rows each): many CTAs per SM
    // overlap one CTA's loads with another's arithmetic
    const long long rows_per_step = 256 / (D / 8);
    auto per_group = [&](long long padded_rows) -> long long {
        if (padded_rows == 0) return 0;
        const long long steps = (padded_rows + rows_per_step - 1) / rows_per_step;
        return (steps + 7) / 8;
    };
    const long long rows_q = a.q != nullptr ? (long long)a.tiles_q * 128 : 0;
    const long long rows_k = a.nkv;
    const long long v_warps = n_grp * (a.nkv / 64) * (D / 32);
    const long long v_ctas = (v_warps + 7) / 8;
    RowJob jq{a.q, a.s, a.qc, a.qs, (unsigned)(a.G * a.nq), (unsigned)a.tiles_q, (unsigned)a.hkv,
              (unsigned)per_group(rows_q)};
    RowJob jk{a.k, a.s_inv, a.kc, a.ks, (unsigned)a.nkv, (unsigned)(a.nkv / 128), (unsigned)a.hkv,
              (unsigned)per_group(rows_k)};
    VJob jv{a.v, a.vtc, a.vts, a.nkv, (unsigned)((a.nkv / 64) * (D / 32))};
    const long long nq = a.q != nullptr ? n_grp * jq.blocks_per_group : 0;
    const long long nk = n_grp * jk.blocks_per_group;
    const long long total = nq + nk + v_ctas;
    if (total > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    quantize_qkv_kernel<T, D><<<(unsigned)total, 256, 0, st>>>(jq, jk, jv, (unsigned)nq, (unsigned)nk,
                                                                (unsigned)v_warps);
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
