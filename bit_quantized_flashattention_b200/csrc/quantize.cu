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

// Rows of Q or K (quantized along D). blockIdx.y is the group: the G*N
// consecutive input rows that share a kv head (G = q heads per kv head for Q,
// 1 for K), padded to whole 128-row tiles; padding rows only receive zero
// scale words. Each lane owns one 8-element chunk of a row (so a warp
// instruction reads 512 contiguous bytes) and walks the group's rows with a
// block stride; its 8 smoothing factors stay in registers. The two halves of a
// 16-element block sit in neighbouring lanes (one shuffle for the maximum), and
// the 4 scale bytes of a 64-element K step are gathered by shuffles into one
// 32-bit word of the MMA-ready atom.
template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, const float* __restrict__ scale,
                                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ sfs,
                                                            unsigned rows_per_group, unsigned tiles_per_group,
                                                            unsigned hkv) {
    constexpr unsigned CPR = D / 8;                        // chunks per row
    constexpr unsigned RPB = 256 / CPR;                    // rows per block step
    constexpr unsigned KS = D / 64;
    __shared__ float lut[128];
    build_rcp_lut(lut);
    const unsigned grp = blockIdx.y;
    const unsigned c = threadIdx.x % CPR;
    const unsigned padded = tiles_per_group * 128;
    float sc[8];
    if (scale != nullptr) {
        const float4* s4 = reinterpret_cast<const float4*>(scale + (size_t)(grp % hkv) * D + c * 8);
        const float4 a = __ldg(s4), b = __ldg(s4 + 1);
        sc[0] = a.x; sc[1] = a.y; sc[2] = a.z; sc[3] = a.w;
        sc[4] = b.x; sc[5] = b.y; sc[6] = b.z; sc[7] = b.w;
    }
    const T* xg = x + (size_t)grp * rows_per_group * D;
    uint8_t* cg = codes + (size_t)grp * rows_per_group * (D / 2);
    uint8_t* sg = sfs + (size_t)grp * tiles_per_group * KS * 512;
    for (unsigned p = blockIdx.x * RPB + threadIdx.x / CPR; p - (threadIdx.x / CPR) < padded;
         p += gridDim.x * RPB) {
        const bool in_tile = p < padded;
        const bool real = p < rows_per_group;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (real) {
            unpack8<T>(*reinterpret_cast<const uint4*>(xg + (size_t)p * D + c * 8), v);
            if (scale != nullptr) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], sc[i]);
            }
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
        // scale word of the 64-element K step: blocks 2k..2k+1 -> byte k
        uint32_t word = ((c & 1u) == 0u) ? (sf << (8u * ((c >> 1) & 3u))) : 0u;
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
        if (in_tile && (c & 7u) == 0u)
            *reinterpret_cast<uint32_t*>(sg + ((size_t)(p >> 7) * KS + c / 8) * 512 + atom_offset(p & 127u)) =
                real ? word : 0u;
    }
}

// ---------------------------------------------------------------------- V

// V quantized along tokens, written transposed. A warp covers 32 channels x 64
// tokens of one group; lane (cc, tb) owns 4 channels (cc = 0..7) x one 16-token
// block (tb = 0..3): it reads 16 rows of 8 bytes (each load instruction reads 4
// rows of 64 contiguous bytes), quantizes one block per channel and writes 8
// code bytes per channel; the 4 scale bytes of a channel for the 64-token half
// come from the lanes tb = 0..3 and are gathered by shuffles. For D = 64 one
// warp per half also fills the padding rows of the scale atoms (row 64 = 1.0
// for the normalizer column of P-Reordering, the rest 0).
template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_v_kernel(const T* __restrict__ v, uint8_t* __restrict__ vtc,
                                                         uint8_t* __restrict__ vts, int nkv) {
    constexpr int NRB = (D + 127) / 128;
    constexpr unsigned CWARPS = D / 32;                    // warps per 64-token half (32 channels each)
    __shared__ float lut[128];
    build_rcp_lut(lut);
    const unsigned lane = threadIdx.x & 31u;
    const unsigned gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // warp within the group
    const unsigned nhalf = (unsigned)nkv / 64u;
    if (gw >= nhalf * CWARPS) return;
    const unsigned grp = blockIdx.y;
    const unsigned cw = gw % CWARPS;
    const unsigned hh = gw / CWARPS;                       // 64-token half over the sequence
    const unsigned cc = lane >> 2, tb = lane & 3u;
    const unsigned d0 = cw * 32 + cc * 4;                  // first channel of this lane
    const unsigned tok0 = hh * 64 + tb * 16;               // first token of this lane's block
    const T* src = v + ((size_t)grp * nkv + tok0) * D + d0;
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
        *reinterpret_cast<uint2*>(vtc + ((size_t)grp * D + d) * (nkv / 2) + tok0 / 2) = make_uint2(lo, hi);
        uint32_t word = sf << (8u * tb);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        if (tb == 0) {
            const size_t atom = (((size_t)grp * (nkv / 128) + j) * NRB + (d >> 7)) * 2 + half;
            *reinterpret_cast<uint32_t*>(vts + atom * 512 + atom_offset(d & 127u)) = word;
        }
    }
    if constexpr (D == 64) {
        if (cw == 0) {
            const size_t atom = ((size_t)grp * (nkv / 128) + j) * 2 + half;
            for (unsigned r = 64 + lane; r < 128; r += 32)
                *reinterpret_cast<uint32_t*>(vts + atom * 512 + atom_offset(r)) = (r == 64) ? 0x38383838u : 0u;
        }
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

template <typename T>
static cudaError_t launch_rows_t(const void* x, const float* scale, uint8_t* codes, uint8_t* sfs, long long n_groups,
                                 int rows_per_group, int tiles_per_group, int hkv, int D, cudaStream_t st) {
    if (n_groups > 65535) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaSuccess;
    switch (D) {
        case 64: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_rows_kernel<T, 64>, 256, 0); break;
        case 128: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_rows_kernel<T, 128>, 256, 0); break;
        default: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_rows_kernel<T, 256>, 256, 0); break;
    }
    if (e != cudaSuccess || occ < 1) occ = 1;
    const long long rows_per_step = 256 / (D / 8);
    const long long steps = ((long long)tiles_per_group * 128 + rows_per_step - 1) / rows_per_step;
    // one resident wave: every CTA of the grid is on an SM at once
    long long bx = ((long long)sms * occ) / n_groups;
    if (bx > steps) bx = steps;
    if (bx < 1) bx = 1;
    const dim3 grid((unsigned)bx, (unsigned)n_groups);
    const T* xp = static_cast<const T*>(x);
    const unsigned rg = (unsigned)rows_per_group, tg = (unsigned)tiles_per_group, hk = (unsigned)hkv;
    switch (D) {
        case 64:
            quantize_rows_kernel<T, 64><<<grid, 256, 0, st>>>(xp, scale, codes, sfs, rg, tg, hk);
            break;
        case 128:
            quantize_rows_kernel<T, 128><<<grid, 256, 0, st>>>(xp, scale, codes, sfs, rg, tg, hk);
            break;
        case 256:
            quantize_rows_kernel<T, 256><<<grid, 256, 0, st>>>(xp, scale, codes, sfs, rg, tg, hk);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_rows(bool bf16, const void* x, const float* scale, uint8_t* codes, uint8_t* sfs,
                                 long long n_groups, int rows_per_group, int tiles_per_group, int hkv, int D,
                                 cudaStream_t st) {
    if (bf16)
        return launch_rows_t<__nv_bfloat16>(x, scale, codes, sfs, n_groups, rows_per_group, tiles_per_group, hkv, D,
                                            st);
    return launch_rows_t<__half>(x, scale, codes, sfs, n_groups, rows_per_group, tiles_per_group, hkv, D, st);
}

template <typename T>
static cudaError_t launch_v_t(const void* v, uint8_t* vtc, uint8_t* vts, long long n_groups, int nkv, int D,
                              cudaStream_t st) {
    if (n_groups > 65535) return cudaErrorInvalidConfiguration;
    const long long warps = (long long)(nkv / 64) * (D / 32);
    const dim3 grid((unsigned)((warps * 32 + 255) / 256), (unsigned)n_groups);
    const T* vp = static_cast<const T*>(v);
    switch (D) {
        case 64:
            quantize_v_kernel<T, 64><<<grid, 256, 0, st>>>(vp, vtc, vts, nkv);
            break;
        case 128:
            quantize_v_kernel<T, 128><<<grid, 256, 0, st>>>(vp, vtc, vts, nkv);
            break;
        case 256:
            quantize_v_kernel<T, 256><<<grid, 256, 0, st>>>(vp, vtc, vts, nkv);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_v(bool bf16, const void* v, uint8_t* vtc, uint8_t* vts, long long n_groups, int nkv, int D,
                              cudaStream_t st) {
    if (bf16) return launch_v_t<__nv_bfloat16>(v, vtc, vts, n_groups, nkv, D, st);
    return launch_v_t<__half>(v, vtc, vts, n_groups, nkv, D, st);
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
