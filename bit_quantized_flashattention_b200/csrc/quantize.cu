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

// Quantize one 16-element block held in registers: returns the scale code,
// writes two 32-bit code words (elements 0-7, 8-15).
__device__ __forceinline__ uint32_t quant_block16(const float (&x)[16], uint32_t& lo, uint32_t& hi) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint32_t sf = cvt_e4m3(__fmul_rn(amax, rn_one_sixth()));
    const float S = e4m3_to_f32(sf);
    const float r = (sf == 0u) ? 0.0f : __frcp_rn(S);
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(x[i], r);
    lo = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    hi = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
    return sf;
}

// Byte offset of (row r, scale k) inside a 512-byte scale atom.
__device__ __forceinline__ uint32_t atom_offset(uint32_t r) { return 16u * (r & 31u) + 4u * ((r >> 5) & 3u); }

// ---------------------------------------------------------------- Q and K

// One thread per 16-element block, consecutive lanes on consecutive blocks so
// that every load and store instruction of a warp covers contiguous bytes.
// Rows are grouped per kv head: a group is G*N consecutive input rows (G = q
// heads per kv head for Q, 1 for K), padded to Tq tiles of 128 rows; threads
// of padding rows only zero their scale byte. The four scale bytes of a
// 64-element K step are gathered with shuffles into one 32-bit word of the
// MMA-ready atom.
template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, const float* __restrict__ scale,
                                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ sfs,
                                                            unsigned total_blocks, unsigned rows_per_group,
                                                            unsigned padded_rows, unsigned hkv) {
    constexpr unsigned NB = D / 16;                        // blocks per row
    constexpr unsigned KS = D / 64;
    const unsigned tid = blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = tid < total_blocks;
    const unsigned kb = tid % NB;
    const unsigned pr = tid / NB;                          // padded row index over all groups
    const unsigned grp = pr / padded_rows;
    const unsigned p = pr - grp * padded_rows;             // row within the group
    const bool real = active && p < rows_per_group;
    uint32_t sf = 0u;
    if (real) {
        const size_t row = (size_t)grp * rows_per_group + p;
        const uint4* src = reinterpret_cast<const uint4*>(x + row * D + kb * 16);
        float v[16], a[8], b[8];
        unpack8<T>(src[0], a);
        unpack8<T>(src[1], b);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] = a[i];
            v[8 + i] = b[i];
        }
        if (scale != nullptr) {
            const float4* sc4 = reinterpret_cast<const float4*>(scale + (size_t)(grp % hkv) * D + kb * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 m = __ldg(sc4 + q);
                v[4 * q + 0] = __fmul_rn(v[4 * q + 0], m.x);
                v[4 * q + 1] = __fmul_rn(v[4 * q + 1], m.y);
                v[4 * q + 2] = __fmul_rn(v[4 * q + 2], m.z);
                v[4 * q + 3] = __fmul_rn(v[4 * q + 3], m.w);
            }
        }
        uint32_t lo, hi;
        sf = quant_block16(v, lo, hi);
        *reinterpret_cast<uint2*>(codes + row * (D / 2) + kb * 8) = make_uint2(lo, hi);
    }
    // gather the 4 scale bytes of this K step (lanes kb&~3 .. kb|3 are adjacent)
    uint32_t w = sf << (8 * (kb & 3));
    w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
    w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
    if (active && (kb & 3) == 0) {
        const unsigned t = p / 128, r = p % 128, s = kb / 4;
        *reinterpret_cast<uint32_t*>(sfs + (((size_t)grp * (padded_rows / 128) + t) * KS + s) * 512 + atom_offset(r)) = w;
    }
}

// ---------------------------------------------------------------------- V

// One CTA per (b*Hkv + g, 128-token tile): stage the tile [128, D] in shared
// memory, then one thread per (channel d, 64-token half) quantizes along tokens
// and writes the transposed codes and one scale word. For D = 64 the extra
// threads fill the atom's padding rows (row 64 = 1.0 for the normalizer
// column of P-Reordering, the rest 0).
template <typename T, int D>
__global__ void __launch_bounds__(2 * (D < 128 ? 128 : D)) quantize_v_kernel(const T* __restrict__ v, uint8_t* __restrict__ vtc,
                                                                           uint8_t* __restrict__ vts, int nkv) {
    constexpr int PITCH = D + 8;                        // elements; keeps column reads conflict-free
    constexpr int NRB = (D + 127) / 128;
    constexpr int NT = 2 * (D < 128 ? 128 : D);
    extern __shared__ __align__(16) uint8_t v_smem[];
    T* tile = reinterpret_cast<T*>(v_smem);
    const int j = blockIdx.x;                           // token tile
    const long long grp = blockIdx.y;                   // b * Hkv + g
    const int ntile = nkv / 128;
    const T* src = v + ((size_t)grp * nkv + (size_t)j * 128) * D;
    constexpr int VEC = 8;                              // elements per 128-bit load
    for (int idx = threadIdx.x; idx < 128 * D / VEC; idx += NT) {
        const int row = idx / (D / VEC), c = idx % (D / VEC);
        const uint4 w = reinterpret_cast<const uint4*>(src + (size_t)row * D)[c];
        *reinterpret_cast<uint4*>(&tile[row * PITCH + c * VEC]) = w;
    }
    __syncthreads();
    const int d = threadIdx.x % (NT / 2);
    const int half = threadIdx.x / (NT / 2);
    const size_t atom = (((size_t)grp * ntile + j) * NRB + (d >> 7)) * 2 + half;
    uint32_t* sf_word = reinterpret_cast<uint32_t*>(vts + atom * 512 + atom_offset((uint32_t)(d & 127)));
    if (d >= D) {                                       // padding rows (only when D = 64)
        *sf_word = (d == D) ? 0x38383838u : 0u;
        return;
    }
    uint32_t words[8];
    uint32_t sfw = 0u;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = to_f32<T>(tile[(half * 64 + blk * 16 + i) * PITCH + d]);
        const uint32_t sf = quant_block16(x, words[2 * blk], words[2 * blk + 1]);
        sfw |= sf << (8 * blk);
    }
    uint4* dst = reinterpret_cast<uint4*>(vtc + ((size_t)grp * D + d) * (nkv / 2) + (size_t)j * 64 + half * 32);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    *sf_word = sfw;
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
    const long long padded = (long long)tiles_per_group * 128;
    const long long total = n_groups * padded * (D / 16);
    if (total > 0xFFFFFFFFLL - 256) return cudaErrorInvalidConfiguration;
    const int threads = 256;
    const unsigned blocks = (unsigned)((total + threads - 1) / threads);
    const T* xp = static_cast<const T*>(x);
    const unsigned tb = (unsigned)total, rg = (unsigned)rows_per_group, pr = (unsigned)padded, hk = (unsigned)hkv;
    switch (D) {
        case 64:
            quantize_rows_kernel<T, 64><<<blocks, threads, 0, st>>>(xp, scale, codes, sfs, tb, rg, pr, hk);
            break;
        case 128:
            quantize_rows_kernel<T, 128><<<blocks, threads, 0, st>>>(xp, scale, codes, sfs, tb, rg, pr, hk);
            break;
        case 256:
            quantize_rows_kernel<T, 256><<<blocks, threads, 0, st>>>(xp, scale, codes, sfs, tb, rg, pr, hk);
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
    const dim3 grid(nkv / 128, (unsigned)n_groups);
    const T* vp = static_cast<const T*>(v);
    const size_t smem = (size_t)128 * (D + 8) * sizeof(T);
    cudaError_t e = cudaSuccess;
    switch (D) {
        case 64:
            quantize_v_kernel<T, 64><<<grid, 256, smem, st>>>(vp, vtc, vts, nkv);
            break;
        case 128:
            quantize_v_kernel<T, 128><<<grid, 256, smem, st>>>(vp, vtc, vts, nkv);
            break;
        case 256:
            e = cudaFuncSetAttribute(quantize_v_kernel<T, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            quantize_v_kernel<T, 256><<<grid, 512, smem, st>>>(vp, vtc, vts, nkv);
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
