// Fused 4-bit attention forward for sm_100a (tcgen05 block-scaled FP4 MMA).
//
// HiFA4 abstract: QK^T and PV both run as 4-bit GEMMs inside FlashAttention,
// the online-softmax state stays in a wider float format, and with
// P-Reordering the softmax normalizer is accumulated from the same quantized
// probabilities P_hat that feed the PV GEMM, fused into that GEMM.
//
// One CTA computes NQT 128-row query tiles (2 for D <= 128, 1 for D = 256) of
// one (batch, kv head) group. A tile's rows are the group's query rows stacked
// head after head (GQA), so a tile may mix heads when Nq is small. Warp roles:
//   warp 0      TMA / bulk-copy producer: Q_hat once, then K_hat and V_hat^T
//               tiles (128 keys) with their scale atoms through shared rings
//   warp 1      TMEM owner; moves the Q scales to TMEM and issues every S MMA
//   warps 2, 3  PV MMA issuers, one per query tile
//   warps 4..   one softmax warpgroup per query tile, thread t owns row t:
//               block maxima of S, running max, P = 2^(S*c - RN(m*c)),
//               P quantized per 16 keys to E2M1 + E4M3 in registers, O rescaled
//               in TMEM when some row's max moved, P_hat codes written to
//               shared memory and their scales to TMEM for the PV MMA.
// The S MMAs run one at a time through one 128-column S buffer in TMEM, in the
// order (kv step 0, query tile 0), (0, 1), (1, 0), ...: once a warpgroup has
// loaded its scores it arrives (without waiting) at its named barrier
// "scores loaded", and the S issuer, blocked in that barrier, issues the next S
// MMA of the order; no warp polls an mbarrier on this path. After the second
// named barrier of the step (P_hat stored, O rescaled) the tile's PV issuer
// issues its PV MMA. An MMA depends only on tcgen05 operations already observed
// complete through an mbarrier, or issued earlier by the same thread.
// With P-Reordering the V tile carries extra rows: a row of E2M1 ones (scale
// 1.0) and zero rows, so the PV MMA (N = D + 8) also produces sum(P_hat) in
// output column D: the normalizer from exactly the codes x scales the MMA used.
//
// Split-kv decode mode (DEC, G*Nq <= 64 query rows per group, D <= 128): the
// kv tiles are cut into 4 contiguous ranges (flash-decoding), all run by one
// CTA. A query tile holds the group's rows twice: lanes 0..63 run range 2x,
// lanes 64..127 range 2x+1 of query tile x. Two zero-padded copies of Q_hat
// (rows in the top half only / in the bottom half only) and two MMAs that
// accumulate into one S give each half its own kv tile; two P_hat buffers with
// the other half zeroed do the same for PV. Each range keeps its own running
// max; at the end the four partial (O, m, l) of a row are merged in shared
// memory with log-sum-exp weights.
//
// TMEM (512 columns): S [0,128), O tiles [128, 128 + NQT*NO), then the
// scale-factor regions of Q, K, P and V.
// Variants by XT: 0 the plain path; 1 also adds a score term per (head, key)
// (the Q-Mean bias); 2 also writes, where asked, each row's P_hat codes and
// scales and its per-tile sums (sum P_hat, sum P) for the epsilon statistics;
// 3 (D = 128, not decode) takes Q unquantized (bf16 / fp16) and quantizes it
// itself: each softmax thread smooths and quantizes its own row into the
// shared-memory Q_hat tile and scale atoms at the start, while the first K / V
// loads are in flight, with the same rule and result as the quantize pass.
//
// Every mbarrier wait is bounded; when one gives up the CTA records
// HIFA4_ERR_TIMEOUT in the workspace, drains its copies and MMAs, frees TMEM
// and exits; the warps then keep meeting at the named barriers (doing no
// work), so every barrier phase still completes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hifa4_device.cuh"
#include "hifa4_kernels.h"

namespace hifa4 {

constexpr int kSmWarp0 = 4;          // first softmax warp (0: loads, 1: TMEM owner + S MMAs, 2-3: PV MMAs)
constexpr int kMaxStages = 12;
constexpr int kDecSplits = 4;        // kv ranges of the split-kv decode mode

template <int D, bool PREORDER, bool DEC, bool QR = false>
struct Cfg {
    static_assert(!DEC || D <= 128, "decode mode needs two query tiles per CTA");
    static constexpr int NQT = D == 256 ? 1 : 2;          // 128-row query tiles per CTA
    // ring slots of K and of V tiles (decode: 4 loads per step; K is read a
    // step before V, so its ring runs further ahead)
    static constexpr int STK = DEC ? 8 : 4;
    static constexpr int STV = DEC ? 8 : 4;
    // every slot of a ring must always hold loads of the same query tile (the
    // empty-barrier parities count that tile's uses of the slot): in decode
    // mode the loads of a step alternate between tiles, so depths are multiples of 4
    static_assert(!DEC || (STK % 4 == 0 && STV % 4 == 0), "ring depth");
    static constexpr int THREADS = 128 + 128 * NQT;
    static constexpr int KS = D / 64;                     // 64-wide K steps of QK^T
    static constexpr int QK_ROW = D / 2;                  // bytes per Q/K row
    static constexpr uint32_t QK_SWZ = D == 64 ? 6u : (D == 128 ? 4u : 2u);   // 32B/64B/128B swizzle
    static constexpr uint32_t QK_SBO = 8u * QK_ROW;       // bytes between 8-row groups
    static constexpr int Q_BYTES = 128 * QK_ROW;
    static constexpr int K_BYTES = 128 * QK_ROW;
    static constexpr int SFQK_BYTES = KS * 512;
    static constexpr int VROWS = D + 16;                  // V^T rows + normalizer block
    static constexpr int V_BYTES = VROWS * 64;
    static constexpr int V_STRIDE = (V_BYTES + 1023) / 1024 * 1024;
    static constexpr int V_TMA_BYTES = D * 64;
    static constexpr int NRB = (D + 127) / 128;           // 128-row blocks of V^T scales
    static constexpr int SFV_BYTES = NRB * 2 * 512;
    static constexpr int P_BYTES = 128 * 64;
    static constexpr int NO = PREORDER ? D + 8 : D;       // accumulator columns per query tile
    static constexpr int NCH = D / 32;                    // 32-column chunks of O
    // scale columns per PV K step: one 4-column block per 128 rows of the B operand
    static constexpr int SFV_PER_KS = 4 * (NRB + ((PREORDER && D >= 128) ? 1 : 0));
    static constexpr int N_SFQ = DEC ? 1 : NQT;           // Q scale regions
    static constexpr int N_SFK = DEC ? 2 : 1;             // K scale regions (decode: one per half)
    static constexpr int N_SFV = DEC ? 2 * NQT : NQT;     // V scale regions
    // TMEM columns
    static constexpr uint32_t COL_S = 0;
    static constexpr uint32_t COL_O = 128;                                // + qt * NO
    static constexpr uint32_t COL_SFQ = COL_O + NQT * NO;
    static constexpr uint32_t COL_SFK = COL_SFQ + N_SFQ * 4 * KS;
    static constexpr uint32_t COL_SFP = COL_SFK + N_SFK * 4 * KS;          // + qt * 8
    static constexpr uint32_t COL_SFV = COL_SFP + NQT * 8;                 // + region * 2 * SFV_PER_KS
    static constexpr uint32_t COL_END = COL_SFV + N_SFV * 2 * SFV_PER_KS;
    static_assert(COL_END <= 512, "TMEM budget");
    // shared memory offsets (operand tiles 1024-aligned)
    static constexpr int OFF_Q = 0;                                       // + buffer * Q_BYTES
    static constexpr int OFF_K = OFF_Q + NQT * Q_BYTES;
    static constexpr int OFF_V = OFF_K + STK * K_BYTES;
    static constexpr int OFF_P = OFF_V + STV * V_STRIDE;                 // + (qt * 2 + buf) * P_BYTES
    static constexpr int OFF_SFQ = OFF_P + NQT * 2 * P_BYTES;             // + qt * SFQK_BYTES
    static constexpr int OFF_SFK = OFF_SFQ + NQT * SFQK_BYTES;
    static constexpr int OFF_SFV = OFF_SFK + STK * SFQK_BYTES;
    static constexpr int OFF_ONES = OFF_SFV + STV * SFV_BYTES;
    static constexpr int OFF_LUT = OFF_ONES + 512;                        // float [128]
    static constexpr int OFF_BAR = OFF_LUT + 128 * 4;
    static constexpr int OFF_BIAS = OFF_BAR + 1024;                      // score-bias staging (XT = 1, 2)
    static constexpr int BIAS_BYTES = 4 * NQT * 2 * 2 * 512;             // per softmax warp: 2 steps x 2 heads x 128 fp32
    static constexpr int OFF_MISC = OFF_BIAS + BIAS_BYTES;
    // in-kernel Q quantization: the caller's bf16 / fp16 Q tiles, two 128-byte
    // column halves per tile (128-byte swizzle), staged by TMA
    static constexpr int QRAW_HALF = 128 * 128;
    static constexpr int OFF_QRAW = (OFF_MISC + 16 + 1023) / 1024 * 1024;  // + (qt * 2 + half) * QRAW_HALF
    static constexpr int SMEM_BYTES = (QR ? OFF_QRAW + NQT * 2 * QRAW_HALF : OFF_MISC + 16) + 1024;   // + alignment slack
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    // decode merge scratch, after the loop: partial O rows (fp32, rows padded by
    // 4 floats) in the K/V ring, the (mc, l) pairs in the P buffers
    static constexpr int MERGE_ROW = D + 4;
    static_assert(!DEC || kDecSplits * 64 * MERGE_ROW * 4 <= OFF_P - OFF_K, "merge scratch");
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kMaxStages];
    uint64_t v_full[kMaxStages];
    uint64_t k_empty[kMaxStages][2];   // K slot no longer read by query tile x's S MMA
    uint64_t v_empty[kMaxStages][2];   // V slot no longer read by query tile x's PV MMA
    uint64_t s_full[2];                // S of query tile x is in TMEM
    uint64_t o_done[2];                // PV MMA of query tile x finished
    uint64_t drain[3];                 // teardown: MMAs issued by the S issuer / each PV issuer
    uint64_t q_ready;                  // in-kernel Q quantization: every softmax thread wrote its Q_hat row
};
static_assert(sizeof(Bars) <= 1024, "barrier area");

#ifndef HIFA4_TRACE_POINT
#define HIFA4_TRACE_POINT(role, j, e)
#endif

__device__ __forceinline__ uint32_t p_swizzle64(uint32_t row, uint32_t chunk) {
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

// Maximum of 16 values held as 8 pairs (three-input max, depth 3).
__device__ __forceinline__ float max16(const float2* v) {
    const float a0 = fmax3f(v[0].x, v[0].y, v[1].x), a1 = fmax3f(v[1].y, v[2].x, v[2].y);
    const float a2 = fmax3f(v[3].x, v[3].y, v[4].x), a3 = fmax3f(v[4].y, v[5].x, v[5].y);
    const float a4 = fmax3f(v[6].x, v[6].y, v[7].x);
    return fmax3f(fmax3f(a0, a1, a2), fmax3f(a3, a4, v[7].y), -INFINITY);
}

// 32 O values (already loaded from TMEM) times alpha, in place.
__device__ __forceinline__ void scale_chunk(uint32_t (&o)[32], float2 a2) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float2 x = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
        o[e] = __float_as_uint(x.x);
        o[e + 1] = __float_as_uint(x.y);
    }
}

// Stores n (a multiple of 8) fp32 values as fp32 / bf16 / fp16 (OUT 2 / 1 / 0).
template <int OUT, int N>
__device__ __forceinline__ void store_out(void* dst, const float* v) {
    if constexpr (OUT == 2) {
        float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < N / 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
        uint32_t w[N / 2];
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if constexpr (OUT == 1) {
                __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                w[i] = *reinterpret_cast<uint32_t*>(&h);
            } else {
                __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
                w[i] = *reinterpret_cast<uint32_t*>(&h);
            }
        }
        uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int i = 0; i < N / 8; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
}

template <int D, bool PREORDER, bool CAUSAL, int OUT, int XT, bool DEC>
__global__ void __launch_bounds__(Cfg<D, PREORDER, DEC>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = Cfg<D, PREORDER, DEC, XT == 3>;
    constexpr int NQT = C::NQT;
    constexpr bool BIAS = XT == 1 || XT == 2;            // score bias
    constexpr bool DIAG = XT == 2;                       // P_hat dump, tile sums
    constexpr bool QRAW = XT == 3;                       // Q quantized in this kernel
    static_assert(!QRAW || (D == 128 && !DEC), "in-kernel Q quantization: D = 128, plain mode");
    constexpr int STK = C::STK, STV = C::STV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* lut = reinterpret_cast<float*>(smem + C::OFF_LUT);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---------------------------------------------------------------- work
    // One work unit = up to NQT consecutive 128-row query tiles of one group
    // (decode: the whole group, whose rows fit in half a tile).
    const int w = blockIdx.x;
    const int units_per_grp = DEC ? 1 : (p.Tq + NQT - 1) / NQT;
    int grp, t0;
    if (!DEC && p.heavy_first) {
        // causal with Nq % (128 * NQT) == 0: units with the most keys first
        const int per_head = p.Nq / (128 * NQT);
        const int per = p.B * p.Hkv * p.G;
        const int u = per_head - 1 - w / per;
        const int rem = w % per;
        grp = rem / p.G;
        t0 = (rem % p.G) * (p.Nq / 128) + u * NQT;
    } else {
        grp = w / units_per_grp;
        t0 = (w % units_per_grp) * NQT;
    }
    const int n_qt = DEC ? NQT : min(NQT, p.Tq - t0);
    const int rows_in_grp = p.G * p.Nq;
    const int T = p.n_kv_tiles;
    // decode: kv range r covers tiles [T*r/4, T*(r+1)/4)
    auto range_begin = [&](int r) -> int { return (int)(((long long)T * r) / kDecSplits); };
    auto range_len = [&](int r) -> int { return range_begin(r + 1) - range_begin(r); };
    // kv tiles each query tile visits (causal: up to the last visible key of its last row)
    auto kv_tiles_of = [&](int qt) -> int {
        if (qt >= n_qt) return 0;
        if (DEC) return max(range_len(2 * qt), range_len(2 * qt + 1));   // steps of the tile
        if (!CAUSAL) return T;
        const int p0 = (t0 + qt) * 128;
        const int p_max = min(p0 + 127, rows_in_grp - 1);
        const int i_max = (p_max / p.Nq == p0 / p.Nq) ? (p_max % p.Nq) : (p.Nq - 1);
        return min(T, (i_max + p.Nkv - p.Nq) / 128 + 1);
    };
    int n_tiles[2];
    n_tiles[0] = kv_tiles_of(0);
    n_tiles[1] = NQT > 1 ? kv_tiles_of(1) : 0;
    const int n_tiles_max = max(n_tiles[0], n_tiles[1]);
    // Loads: one kv tile (K and V) each, in consumption order. Plain mode:
    // load j = kv tile j for the tiles visiting it; decode: load 4t + 2x + h =
    // step t of range 2x + h (a null load past the end of a shorter range).
    const int n_loads = DEC ? 4 * n_tiles_max : n_tiles_max;
    auto load_tile = [&](int i) -> int { return DEC ? range_begin(i & 3) + (i >> 2) : i; };
    auto load_users = [&](int i) -> int {   // bit x: query tile x reads this load
        if (DEC) return (i >> 2) < range_len(i & 3) ? 1 << ((i & 3) >> 1) : 0;
        return (i < n_tiles[0] ? 1 : 0) | (NQT > 1 && i < n_tiles[1] ? 2 : 0);
    };

    // The S MMAs run one at a time through the one S buffer, in the order
    // (step 0, query tile 0), (0, 1), (1, 0), (1, 1), ... skipping the steps a
    // query tile does not take. The item after (j, x) in that order:
    auto next_item = [&](int j, int x, int& nj, int& nx) -> bool {
#pragma unroll 1
        for (int guard = 0; guard < 2 * NQT + 2; ++guard) {
            if (++x >= NQT) { x = 0; ++j; }
            if (j >= n_tiles_max) return false;
            if (j < n_tiles[x]) { nj = j; nx = x; return true; }
        }
        return false;
    };

    // One load of the K or V ring (a null load, which nothing reads, only
    // arrives on its barrier); issued by the producer thread alone.
    auto issue_k = [&](int i) {
        const int st = i % STK;
        if (load_users(i) == 0) {
            mbar_arrive(&bars->k_full[st]);
            return;
        }
        const int j = load_tile(i);
        mbar_arrive_expect_tx(&bars->k_full[st], C::K_BYTES + C::SFQK_BYTES);
        tma_load_2d(smem + C::OFF_K + st * C::K_BYTES, &tmK, 0, grp * p.Nkv + j * 128, &bars->k_full[st]);
        bulk_load(smem + C::OFF_SFK + st * C::SFQK_BYTES, p.ks + ((size_t)grp * T + j) * C::SFQK_BYTES,
                  C::SFQK_BYTES, &bars->k_full[st]);
    };
    auto issue_v = [&](int i) {
        const int st = i % STV;
        if (load_users(i) == 0) {
            mbar_arrive(&bars->v_full[st]);
            return;
        }
        const int j = load_tile(i);
        mbar_arrive_expect_tx(&bars->v_full[st], C::V_TMA_BYTES + C::SFV_BYTES);
        tma_load_2d(smem + C::OFF_V + st * C::V_STRIDE, &tmV, 0, (grp * T + j) * D, &bars->v_full[st]);
        bulk_load(smem + C::OFF_SFV + st * C::SFV_BYTES, p.vts + ((size_t)grp * T + j) * C::SFV_BYTES,
                  C::SFV_BYTES, &bars->v_full[st]);
    };
    int ik = 0, iv = 0;                     // K / V loads issued so far (producer thread)

    // --------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        HIFA4_TRACE_POINT(4, 63, 0);
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_ready, 128 * NQT);
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            for (int x = 0; x < 2; ++x) {
                mbar_init(&bars->k_empty[s][x], 1);
                mbar_init(&bars->v_empty[s][x], 1);
            }
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->o_done[x], 1);
        }
        for (int k = 0; k < 3; ++k) mbar_init(&bars->drain[k], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x >= 128 && threadIdx.x < 256) {
        const uint32_t i = threadIdx.x - 128;
        lut[i] = (i == 0) ? 0.0f : __frcp_rn(e4m3_to_f32(i));
        // normalizer block of V^T (rows D..D+15 of every stage): one row of E2M1
        // ones (code 2 in both nibbles), zero rows; and the scale atom of the
        // ones row (row 0 of an atom = 1.0) used when D >= 128.
        for (int s = 0; s < STV; ++s) {
            uint32_t* row = reinterpret_cast<uint32_t*>(smem + C::OFF_V + s * C::V_STRIDE + D * 64);
            for (int k = i; k < 16 * 16; k += 128) row[k] = (k < 16) ? 0x22222222u : 0u;
        }
        reinterpret_cast<uint32_t*>(smem + C::OFF_ONES)[i] = (i == 0) ? 0x38383838u : 0u;
    }
    if constexpr (DEC) {
        // the P_hat buffers: a thread only ever writes its own row, in the
        // buffer of its half, so the other half of every buffer stays zero
        if (threadIdx.x >= 128) {
            uint4* pz = reinterpret_cast<uint4*>(smem + C::OFF_P);
            for (int k = threadIdx.x - 128; k < NQT * 2 * C::P_BYTES / 16; k += 128 * NQT) pz[k] = make_uint4(0, 0, 0, 0);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

    // Scale atoms moved shared->TMEM, and the MMAs. An MMA is issued only after
    // every tcgen05 operation it depends on has completed (observed through an
    // mbarrier), or was issued earlier by the same thread (one thread's
    // tcgen05 operations run in issue order).
    // Shared-memory descriptors: a base descriptor plus (byte offset >> 4) in
    // the 14-bit address field (all shared addresses are below 256 KB).
    const uint32_t idesc_s = idesc_fp4_block16(128);
    auto sf_desc = [&](uint32_t off) { return smem_desc(sbase + off, 0u, 128u, 0u); };
    const uint64_t qk_desc0 = smem_desc(sbase, 16u, C::QK_SBO, C::QK_SWZ);
    const uint64_t pv_desc0 = smem_desc(sbase, 16u, 512u, 4u);
    // last query tile (in S order) that visits plain-mode kv tile j
    auto last_x_of = [&](int j) -> int { return (NQT > 1 && j < n_tiles[1]) ? 1 : 0; };
    auto copy_sfk = [&](int li, int region) {
        const int st = li % STK;
#pragma unroll
        for (int s = 0; s < C::KS; ++s)
            tmem_cp_scale_atom(tmem + C::COL_SFK + region * 4 * C::KS + 4 * s,
                               sf_desc(C::OFF_SFK + st * C::SFQK_BYTES + 512 * s));
    };
    auto copy_sfv = [&](int li, int region) {
        const int st = li % STV;
        const uint32_t sfv = C::OFF_SFV + st * C::SFV_BYTES;
        const uint32_t col = C::COL_SFV + region * 2 * C::SFV_PER_KS;
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int rb = 0; rb < C::NRB; ++rb)
                tmem_cp_scale_atom(tmem + col + s * C::SFV_PER_KS + 4 * rb, sf_desc(sfv + (rb * 2 + s) * 512));
    };
    // the K scales an item needs next (plain: the next kv tile, after the last
    // item on this one; decode: the two loads of the next item), moved in by the
    // S issuer right after the current MMAs. Returns false if a load never came.
    auto prefetch_sfk = [&](int j, int x) -> bool {
        int nj, nx;
        if (!next_item(j, x, nj, nx)) return true;
        if constexpr (DEC) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int li = 4 * nj + 2 * nx + h;
                if (!(load_users(li) & (1 << nx))) continue;
                if (!mbar_wait_poll(&bars->k_full[li % STK], (li / STK) & 1, ctl, 32)) return false;
                copy_sfk(li, h);
            }
        } else {
            if (nj == j) return true;
            if (!mbar_wait_poll(&bars->k_full[nj % STK], (nj / STK) & 1, ctl, 32)) return false;
            copy_sfk(nj, 0);
        }
        return true;
    };
    // S = Q_hat K_hat^T of item (j, x): one MMA per half (decode: Q_hat copy h
    // against range 2x+h's kv tile, accumulating into the same S).
    auto issue_s = [&](int j, int x) -> bool {
        bool first = true;
#pragma unroll
        for (int h = 0; h < (DEC ? 2 : 1); ++h) {
            const int li = DEC ? 4 * j + 2 * x + h : j;
            if (DEC && !(load_users(li) & (1 << x))) continue;
            const int st = li % STK;
            const uint64_t kd = qk_desc0 + ((C::OFF_K + st * C::K_BYTES) >> 4);
            const uint64_t qd = qk_desc0 + ((C::OFF_Q + (DEC ? h : x) * C::Q_BYTES) >> 4);
            const uint32_t sfq = tmem + C::COL_SFQ + (DEC ? 0 : x) * 4 * C::KS;
            const uint32_t sfk = tmem + C::COL_SFK + (DEC ? h : 0) * 4 * C::KS;
#pragma unroll
            for (int s = 0; s < C::KS; ++s)
                mma_fp4_block16(tmem + C::COL_S, qd + 2 * s, kd + 2 * s, idesc_s, sfq + 4 * s, sfk + 4 * s,
                                (first && s == 0) ? 0u : 1u);
            first = false;
        }
        tc_commit(&bars->s_full[x]);
#pragma unroll
        for (int h = 0; h < (DEC ? 2 : 1); ++h) {
            const int li = DEC ? 4 * j + 2 * x + h : j;
            if (load_users(li) & (1 << x)) tc_commit(&bars->k_empty[li % STK][x]);
        }
        if (!DEC && !(x == last_x_of(j))) return true;
        return prefetch_sfk(j, x);
    };
    // O(x) += P_hat V_hat of step j (decode: one MMA per half), then the V
    // scales of the next step are moved in for the next PV MMA of this tile.
    auto issue_pv = [&](int j, int x) -> bool {
        const uint32_t o = tmem + C::COL_O + x * C::NO;
        bool first = j == 0;
#pragma unroll
        for (int h = 0; h < (DEC ? 2 : 1); ++h) {
            const int li = DEC ? 4 * j + 2 * x + h : j;
            if (DEC && !(load_users(li) & (1 << x))) continue;
            const int st = li % STV;
            const uint64_t vd = pv_desc0 + ((C::OFF_V + st * C::V_STRIDE) >> 4);
            const uint64_t pd = pv_desc0 + ((C::OFF_P + (x * 2 + (DEC ? h : (j & 1))) * C::P_BYTES) >> 4);
            const uint32_t col_sfv = C::COL_SFV + (DEC ? 2 * x + h : x) * 2 * C::SFV_PER_KS;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t acc = (first && s == 0) ? 0u : 1u;
                const uint32_t sfa = tmem + C::COL_SFP + x * 8 + 4 * s;
                const uint32_t sfb = tmem + col_sfv + s * C::SFV_PER_KS;
                if constexpr (D == 256 && PREORDER) {
                    mma_fp4_block16(o, pd + 2 * s, vd + 2 * s, idesc_fp4_block16(128), sfa, sfb, acc);
                    mma_fp4_block16(o + 128, pd + 2 * s, vd + ((128 * 64) >> 4) + 2 * s, idesc_fp4_block16(C::NO - 128),
                                    sfa, sfb + 4, acc);
                } else {
                    mma_fp4_block16(o, pd + 2 * s, vd + 2 * s, idesc_fp4_block16(C::NO), sfa, sfb, acc);
                }
            }
            first = false;
        }
        tc_commit(&bars->o_done[x]);
#pragma unroll
        for (int h = 0; h < (DEC ? 2 : 1); ++h) {
            const int li = DEC ? 4 * j + 2 * x + h : j;
            if (load_users(li) & (1 << x)) tc_commit(&bars->v_empty[li % STV][x]);
        }
        if (j + 1 < n_tiles[x]) {
#pragma unroll
            for (int h = 0; h < (DEC ? 2 : 1); ++h) {
                const int li = DEC ? 4 * (j + 1) + 2 * x + h : j + 1;
                if (!(load_users(li) & (1 << x))) continue;
                if (!mbar_wait_poll(&bars->v_full[li % STV], (li / STV) & 1, ctl, 32)) return false;
                copy_sfv(li, DEC ? 2 * x + h : x);
            }
        }
        return true;
    };

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // The set-up above overlaps the end of the previous kernel in the
        // stream (programmatic dependent launch); the packed operands are read
        // only after it has completed. Every other read of those operands
        // goes through this warp's copies. A slot is refilled once every query
        // tile that read the previous load in it has released it.
        grid_dependency_wait();
        if (lane == 0 && !p.stall_loads) {
            const int nq_load = QRAW ? 0 : (DEC ? 1 : n_qt);
            if constexpr (QRAW) {
                // the caller's Q tiles (rows of D = 128 bf16 / fp16, 256 bytes) as
                // two 128-byte column halves each; rows past the tensor read as 0
                mbar_arrive_expect_tx(&bars->q_full, n_qt * 2 * C::QRAW_HALF);
                for (int qt = 0; qt < n_qt; ++qt)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d(smem + C::OFF_QRAW + (qt * 2 + h) * C::QRAW_HALF, &tmQ, 128 * h,
                                    grp * rows_in_grp + (t0 + qt) * 128, &bars->q_full);
            } else {
                mbar_arrive_expect_tx(&bars->q_full, nq_load * (C::Q_BYTES + C::SFQK_BYTES));
            }
            for (int qt = 0; qt < nq_load; ++qt) {
                tma_load_2d(smem + C::OFF_Q + qt * C::Q_BYTES, &tmQ, 0, grp * rows_in_grp + (t0 + qt) * 128,
                            &bars->q_full);
                bulk_load(smem + C::OFF_SFQ + qt * C::SFQK_BYTES,
                          p.qs + ((size_t)grp * p.Tq + t0 + qt) * C::SFQK_BYTES, C::SFQK_BYTES, &bars->q_full);
            }
            // K and V go through their rings independently: a K slot is free
            // once the S MMAs that read it finished, a V slot once the PV MMAs
            // did, so K runs a step further ahead than V needs to.
            auto slot_free = [&](uint64_t (*empty)[2], int i, int stages) -> bool {
                const int ip = i - stages;                           // previous load in this slot
                if (ip < 0) return true;
                const int users = load_users(ip);
                const uint32_t ph = (ip / stages) & 1;
                for (int x = 0; x < NQT; ++x)
                    if (((users >> x) & 1) && !mbar_test(&empty[ip % stages][x], ph)) return false;
                return true;
            };
            bool ok = true;
            // start of the current run of iterations without progress (0: none);
            // the timer is read only while idle (a read costs hundreds of cycles)
            uint64_t t_idle = 0;
            while ((ik < n_loads || iv < n_loads) && ok) {
                bool progressed = false;
                if (ik < n_loads && slot_free(bars->k_empty, ik, STK)) {
                    issue_k(ik);
                    HIFA4_TRACE_POINT(4, ik, 1);
                    ++ik;
                    progressed = true;
                }
                if (iv < n_loads && slot_free(bars->v_empty, iv, STV)) {
                    issue_v(iv);
                    ++iv;
                    progressed = true;
                }
                if (progressed) {
                    t_idle = 0;
                } else {
                    __nanosleep(128);
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0) t_idle = now;
                    if (*abort_flag) {
                        ok = false;
                    } else if (now - t_idle > p.wait_limit_ns) {
                        *abort_flag = 1;
                        atomicExch(p.status, kStatusTimeout);
                        ok = false;
                    }
                }
            }
            if (!ok) {
                // drain the copies still in flight before the CTA exits
                for (int i = max(0, ik - STK); i < ik; ++i)
                    mbar_wait_drain(&bars->k_full[i % STK], (i / STK) & 1, p.wait_limit_ns);
                for (int i = max(0, iv - STV); i < iv; ++i)
                    mbar_wait_drain(&bars->v_full[i % STV], (i / STV) & 1, p.wait_limit_ns);
                mbar_wait_drain(&bars->q_full, 0, p.wait_limit_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- S issuer
        // Moves the Q scales (and the first step's K and V scales) to TMEM,
        // issues the first S MMA, then walks the S order: once the consumer of
        // an S tile has loaded it (named barrier "scores loaded" of that
        // warpgroup, which arrives without waiting) the next S MMA is issued.
        // A warp blocked in a named barrier takes no issue slots.
        bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(QRAW ? &bars->q_ready : &bars->q_full, 0, ctl));
        int j = 0, x = 0;
        bool more = next_item(0, -1, j, x);
        // the loads the first step reads (plain: load 0; decode: loads 0..3)
        for (int i = 0; i < (DEC ? 4 : 1) && ok && more; ++i) {
            if (load_users(i) == 0) continue;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->k_full[i % STK], 0, ctl));
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->v_full[i % STV], 0, ctl));
        }
        if constexpr (DEC) {
            if (ok) {
                // Q_hat copy 0 = the group's rows in the top half (rows past
                // them zeroed); copy 1 = the same rows in the bottom half. Rows r
                // and r + 64 share their swizzle phase, so rows move as bytes.
                const int nrow = rows_in_grp;                            // <= 64
                uint4* q0 = reinterpret_cast<uint4*>(smem + C::OFF_Q);
                uint4* q1 = reinterpret_cast<uint4*>(smem + C::OFF_Q + C::Q_BYTES);
                constexpr int PER_ROW = C::QK_ROW / 16;
                for (int k = lane; k < 128 * PER_ROW; k += 32) {
                    const int r = k / PER_ROW;
                    q1[k] = (r >= 64 && r - 64 < nrow) ? q0[k - 64 * PER_ROW] : make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                for (int k = lane; k < 128 * PER_ROW; k += 32)
                    if (k / PER_ROW >= nrow) q0[k] = make_uint4(0, 0, 0, 0);
                // Q scales: rows r + 64 and r + 96 of each atom take rows r and
                // r + 32 (bytes 8..15 of a 16-byte atom row = bytes 0..7)
                for (int a = 0; a < C::KS; ++a) {
                    uint2* row = reinterpret_cast<uint2*>(smem + C::OFF_SFQ + a * 512 + 16 * lane);
                    row[1] = row[0];
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
        }
        bool issued_any = false;
        if (ok) {
            tc_fence_after();
            if (lane == 0) {
                for (int qt = 0; qt < C::N_SFQ; ++qt) {
#pragma unroll
                    for (int s = 0; s < C::KS; ++s)
                        tmem_cp_scale_atom(tmem + C::COL_SFQ + qt * 4 * C::KS + 4 * s,
                                           sf_desc(C::OFF_SFQ + qt * C::SFQK_BYTES + 512 * s));
                }
                for (int rg = 0; rg < C::N_SFV; ++rg) {
                    // scale atom of the normalizer rows (rows D.. of the V operand)
                    if constexpr (PREORDER && D >= 128) {
#pragma unroll
                        for (int s = 0; s < 2; ++s)
                            tmem_cp_scale_atom(tmem + C::COL_SFV + rg * 2 * C::SFV_PER_KS + s * C::SFV_PER_KS + 4 * C::NRB,
                                               sf_desc(C::OFF_ONES));
                    }
                }
                if (more) {
                    if constexpr (DEC) {
                        for (int i = 0; i < 4; ++i) {
                            if (load_users(i) == 0) continue;
                            if (i < 2) copy_sfk(i, i);
                            copy_sfv(i, i);
                        }
                    } else {
                        copy_sfk(0, 0);
                        for (int qt = 0; qt < n_qt; ++qt) copy_sfv(0, qt);
                    }
                    (void)issue_s(j, x);
                    issued_any = true;
                }
            }
            __syncwarp();
        }
        // every S tile's consumer arrives once at its barrier, also after a
        // failure, so this walk always runs to the end of the order
        while (more) {
            named_barrier_sync(1 + 2 * x, 160);
            HIFA4_TRACE_POINT(2, j, 2 * x);
            int nj = 0, nx = 0;
            more = next_item(j, x, nj, nx);
            if (more && lane == 0 && !*abort_flag) {
                tc_fence_after();
                (void)issue_s(nj, nx);
                issued_any = true;
            }
            __syncwarp();
            HIFA4_TRACE_POINT(2, j, 2 * x + 1);
            j = nj;
            x = nx;
        }
        // wait until every MMA / copy this warp issued has finished
        if (lane == 0 && issued_any) {
            tc_commit(&bars->drain[0]);
            mbar_wait_drain(&bars->drain[0], 0, p.wait_limit_ns);
        }
        __syncwarp();
    } else if (warp == 2 || (warp == 3 && NQT > 1)) {
        // ----------------------------------------------------- PV issuers
        // One warp per query tile: once the tile's P_hat is stored and its O
        // rescaled (named barrier "P stored"), it issues the PV MMA.
        const int qt = warp - 2;
        bool issued_any = false;
        // the warpgroup arrives on every step, also after a failure
        for (int jj = 0; jj < n_tiles[qt]; ++jj) {
            named_barrier_sync(2 + 2 * qt, 160);
            if (lane == 0 && !*abort_flag) {
                tc_fence_after();
                (void)issue_pv(jj, qt);
                issued_any = true;
            }
            __syncwarp();
            HIFA4_TRACE_POINT(3, jj, 1 + qt);
        }
        // wait until every MMA this warp issued has finished before TMEM is freed
        if (lane == 0 && issued_any) {
            tc_commit(&bars->drain[1 + qt]);
            mbar_wait_drain(&bars->drain[1 + qt], 0, p.wait_limit_ns);
        }
        __syncwarp();
    } else if (warp >= kSmWarp0) {
        // ------------------------------------------------------------ softmax
        const int qt = (warp - kSmWarp0) >> 2;             // query tile of this warpgroup
        const int wq = warp & 3;                           // TMEM lane quarter
        const uint32_t id_s = 1 + 2 * qt, id_p = 2 + 2 * qt;     // shared with the S issuer / the tile's PV issuer
        const int row = wq * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tO = tl + C::COL_O + qt * C::NO;
        const int half = DEC ? row >> 6 : 0;               // decode: which kv range of the tile
        const int range = 2 * qt + half;
        const int prow = DEC ? (row & 63) : (t0 + qt) * 128 + row;   // row within the group
        const bool valid = qt < n_qt && prow < rows_in_grp;
        const int qi = prow % p.Nq;
        const int last = valid ? (CAUSAL ? qi + p.Nkv - p.Nq : p.Nkv - 1) : -1;
        const size_t out_row = (size_t)grp * rows_in_grp + prow;
        const int nt = n_tiles[qt];
        const int own_steps = DEC ? range_len(range) : nt;
        const int kt0 = DEC ? range_begin(range) : 0;
        const float c = p.c;
        const float2 c2 = make_float2(c, c);
        const float one_sixth = rn_one_sixth();
        const uint32_t lut_s = smem_u32(lut);
        float m_old = -INFINITY, mc_old = 0.0f, l_hp = 0.0f;
        bool ok = true;                                     // false once a wait gave up (then no more work)
        if constexpr (QRAW) {
            // this row of the query tile, from the caller's Q staged in shared
            // memory: RN(x * s), per 16 elements sf = E4M3(amax * RN(1/6)), codes
            // E2M1(RN(x * RN(1/sf))) (the quantize pass's rule), into the Q_hat
            // tile (64-byte K-major rows, 64B swizzle) and the MMA-ready scale
            // atoms; then arrive on q_ready (also after a failed wait).
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->q_full, 0, ctl));
            HIFA4_TRACE_POINT(qt, 61, 0);
            uint32_t w[16];
            uint32_t sfa[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = 0u;
            if (ok && valid) {
                // the smoothing factors may come from the previous kernel of the
                // stream: read them only once it has completed
                if (p.q_scale != nullptr) grid_dependency_wait();
                const float* sc = p.q_scale != nullptr ? p.q_scale + (size_t)(grp % p.Hkv) * D : nullptr;
#pragma unroll
                for (int half = 0; half < 2; ++half) {   // 64 elements (4 blocks) at a time
                    // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
                    const uint32_t rb = sbase + C::OFF_QRAW + (qt * 2 + half) * C::QRAW_HALF + row * 128;
                    uint4 raw[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 f4 = lds_v4f(rb + ((c ^ (row & 7)) << 4));
                        raw[c] = make_uint4(__float_as_uint(f4.x), __float_as_uint(f4.y), __float_as_uint(f4.z),
                                            __float_as_uint(f4.w));
                    }
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) {
                        const int b = 4 * half + bb;
                        float x[16];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t* u = reinterpret_cast<const uint32_t*>(&raw[2 * bb + h]);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 f;
                                if (p.q_bf16) {
                                    f = make_float2(__uint_as_float(u[e] << 16), __uint_as_float(u[e] & 0xFFFF0000u));
                                } else {
                                    f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
                                }
                                x[8 * h + 2 * e] = f.x;
                                x[8 * h + 2 * e + 1] = f.y;
                            }
                        }
                        if (sc != nullptr) {
                            const float4* s4 = reinterpret_cast<const float4*>(sc + 16 * b);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 v = __ldg(s4 + q);
                                x[4 * q] = __fmul_rn(x[4 * q], v.x);
                                x[4 * q + 1] = __fmul_rn(x[4 * q + 1], v.y);
                                x[4 * q + 2] = __fmul_rn(x[4 * q + 2], v.z);
                                x[4 * q + 3] = __fmul_rn(x[4 * q + 3], v.w);
                            }
                        }
                        float amax = 0.0f;
#pragma unroll
                        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
                        const uint32_t sf = cvt_e4m3(__fmul_rn(amax, rn_one_sixth()));
                        const float r = lds_f32(smem_u32(lut) + 4u * (sf & 127u));
                        float y[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(x[e], r);
                        w[2 * b] = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
                        w[2 * b + 1] = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
                        sfa[b >> 2] |= sf << (8 * (b & 3));
                    }
                }
            }
            const uint32_t qb = sbase + C::OFF_Q + qt * C::Q_BYTES;
#pragma unroll
            for (int q = 0; q < 4; ++q) sts_v4(qb + p_swizzle64(row, q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            const uint32_t ao = 16u * (row & 31) + 4u * (row >> 5);       // row's word in a scale atom
#pragma unroll
            for (int a = 0; a < 2; ++a) sts_u32(sbase + C::OFF_SFQ + qt * C::SFQK_BYTES + 512 * a + ao, sfa[a]);
            fence_proxy_async_smem();
            mbar_arrive(&bars->q_ready);
            HIFA4_TRACE_POINT(qt, 61, 1);
        }
        // XT = 1, 2: the score bias of a step's kv tile is staged in shared memory
        // one step ahead, a warp at a time: lane l loads 4 of the 128 values of
        // each head the warp's rows belong to (at most two: Nq >= 16), and every
        // row then reads its head's 128 values back as broadcast loads.
        const bool use_bias = BIAS && p.s_bias != nullptr;
        const int my_head = valid ? (int)(out_row / (size_t)p.Nq) : -1;
        const int head0 = __shfl_sync(0xFFFFFFFFu, my_head, 0);
        const int head1 = __reduce_max_sync(0xFFFFFFFFu, my_head);
        const uint32_t bias_s = sbase + C::OFF_BIAS + (uint32_t)(warp - kSmWarp0) * 2048u;   // [step & 1][head 0/1][128]
        float4 bias_next[2];
        auto load_bias = [&](int jn) {                      // this lane's part of step jn's rows
            if (use_bias && head0 >= 0 && jn < own_steps) {
                const size_t col = (size_t)(kt0 + jn) * 128 + 4 * lane;
                bias_next[0] = __ldg(reinterpret_cast<const float4*>(p.s_bias + (size_t)head0 * p.Nkv + col));
                bias_next[1] = head1 != head0
                                   ? __ldg(reinterpret_cast<const float4*>(p.s_bias + (size_t)head1 * p.Nkv + col))
                                   : bias_next[0];
            }
        };
        auto stage_bias = [&](int jn) {
            if (use_bias && head0 >= 0 && jn < own_steps) {
                __syncwarp();
                const uint32_t b = bias_s + (uint32_t)(jn & 1) * 1024u + 16u * lane;
                sts_v4(b, __float_as_uint(bias_next[0].x), __float_as_uint(bias_next[0].y),
                       __float_as_uint(bias_next[0].z), __float_as_uint(bias_next[0].w));
                sts_v4(b + 512u, __float_as_uint(bias_next[1].x), __float_as_uint(bias_next[1].y),
                       __float_as_uint(bias_next[1].z), __float_as_uint(bias_next[1].w));
                __syncwarp();
            }
        };
        if constexpr (BIAS) {
            // the bias is written by the previous kernel of the stream: read it
            // only once that kernel has completed (programmatic dependent launch)
            if (use_bias) grid_dependency_wait();
            load_bias(0);
            stage_bias(0);
        }
        for (int j = 0; j < nt; ++j) {
            HIFA4_TRACE_POINT(qt, j, 0);
            ok = __all_sync(0xFFFFFFFFu, ok && mbar_wait(&bars->s_full[qt], j & 1, ctl));
            HIFA4_TRACE_POINT(qt, j, 1);
            // (loaded even when the wait gave up: stale values, discarded below)
            float2 S[64];
            {
                tc_fence_after();
                uint32_t r[128];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld32(tl + C::COL_S + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * q));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 64; ++e) S[e] = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                tc_fence_before();
            }
            // every row has its scores: the S buffer is free for the next S MMA.
            // Arriving without waiting is safe while the waits succeed (this
            // warpgroup cannot reach the next step's arrival before the issuer
            // has passed this barrier: that S MMA is issued after it); after a
            // failure the waits no longer hold it back, so it syncs instead.
            if (ok) named_barrier_arrive(id_s, 160); else named_barrier_sync(id_s, 160);
            HIFA4_TRACE_POINT(qt, j, 2);
            if (ok) {
                // this row's kv tile of the step; keys past `last` are masked
                // (decode: a row whose range has ended masks the whole step)
                const int n0 = (kt0 + j) * 128;
                const int lim = j < own_steps ? last : -1;
                if constexpr (BIAS) {
                    load_bias(j + 1);
                    if (use_bias && my_head >= 0 && j < own_steps) {
                        const uint32_t bp = bias_s + (uint32_t)(j & 1) * 1024u + (my_head != head0 ? 512u : 0u);
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float4 b4 = lds_v4f(bp + 16u * e);
                            S[2 * e] = make_float2(__fadd_rn(S[2 * e].x, b4.x), __fadd_rn(S[2 * e].y, b4.y));
                            S[2 * e + 1] = make_float2(__fadd_rn(S[2 * e + 1].x, b4.z), __fadd_rn(S[2 * e + 1].y, b4.w));
                        }
                    }
                }
                if (n0 + 127 > lim) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        if (n0 + 2 * e > lim) S[e].x = -INFINITY;
                        if (n0 + 2 * e + 1 > lim) S[e].y = -INFINITY;
                    }
                }
                // block maxima of S (they also give the block maxima of P: 2^x is monotone)
                float bm[8];
#pragma unroll
                for (int b = 0; b < 8; ++b) bm[b] = max16(S + 8 * b);
                const float mx = fmax3f(fmax3f(bm[0], bm[1], bm[2]), fmax3f(bm[3], bm[4], bm[5]), fmaxf(bm[6], bm[7]));
                const float m_new = fmaxf(m_old, mx);
                const float mc_new = (m_new == -INFINITY) ? 0.0f : __fmul_rn(m_new, c);
                const float alpha = (m_old == -INFINITY) ? 0.0f : ex2_approx(mc_old - mc_new);
                const float2 nmc2 = make_float2(-mc_new, -mc_new);
                // P = 2^(S*c - mc) in place: one stream of independent FFMA2 +
                // ex2 pairs that keeps the MUFU busy; then 8 blocks of 16 keys to
                // E4M3 scales and E2M1 codes (no MUFU on that chain but the 8
                // block-scale exponentials)
                float2 lsum2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const float2 t = __ffma2_rn(S[e], c2, nmc2);
                    S[e] = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                    if constexpr (!PREORDER || DIAG) lsum2 = __fadd2_rn(lsum2, S[e]);
                }
                uint32_t code[16];
                uint32_t sfw[2] = {0u, 0u};
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const float pm = ex2_approx(__fmaf_rn(bm[b], c, -mc_new));
                    const uint32_t sf = cvt_e4m3(__fmul_rn(pm, one_sixth));
                    const float r = lds_f32(lut_s + 4u * (sf & 127u));
                    const float2 r2 = make_float2(r, r);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 yy = __fmul2_rn(S[8 * b + 4 * h + e], r2);
                            y[2 * e] = yy.x;
                            y[2 * e + 1] = yy.y;
                        }
                        code[2 * b + h] = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
                    }
                    sfw[b >> 2] |= sf << (8 * (b & 3));
                }
                HIFA4_TRACE_POINT(qt, j, 3);
                // rescale O of this tile's rows when some row's max moved (the
                // previous PV must be done); two 32-column chunks in flight at a time
                if (j > 0) {
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_done[qt], (j - 1) & 1, ctl));
                    HIFA4_TRACE_POINT(qt, j, 4);
                    if (ok) {
                        tc_fence_after();
                        if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
                            const float2 a2 = make_float2(alpha, alpha);
                            uint32_t lv = 0;
                            if constexpr (PREORDER) tmem_ld1(tO + D, lv);
#pragma unroll
                            for (int ch = 0; ch < C::NCH; ch += 2) {
                                uint32_t o0[32], o1[32];
                                tmem_ld32(tO + 32 * ch, o0);
                                if (ch + 1 < C::NCH) tmem_ld32(tO + 32 * (ch + 1), o1);
                                tmem_wait_ld_dep(o0);
                                if (ch + 1 < C::NCH) tmem_wait_ld_dep(o1);
                                scale_chunk(o0, a2);
                                tmem_st32(tO + 32 * ch, o0);
                                if (ch + 1 < C::NCH) {
                                    scale_chunk(o1, a2);
                                    tmem_st32(tO + 32 * (ch + 1), o1);
                                }
                            }
                            if constexpr (PREORDER) tmem_st1(tO + D, __float_as_uint(__fmul_rn(__uint_as_float(lv), alpha)));
                            tmem_wait_st();
                        }
                    }
                }
                HIFA4_TRACE_POINT(qt, j, 5);
                if constexpr (!PREORDER) l_hp = __fmaf_rn(alpha, l_hp, lsum2.x + lsum2.y);
                {
                    const uint32_t pb = sbase + C::OFF_P + (qt * 2 + (DEC ? half : (j & 1))) * C::P_BYTES;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        sts_v4(pb + p_swizzle64(row, q), code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
                    // the row's E4M3 scales straight into the TMEM column the PV MMA
                    // reads for it (row r: lane r, column base + r/32 of each K step;
                    // the previous PV, the last reader, is done)
                    tmem_st1(tl + C::COL_SFP + qt * 8 + wq, sfw[0]);
                    tmem_st1(tl + C::COL_SFP + qt * 8 + 4 + wq, sfw[1]);
                    tmem_wait_st();
                    if constexpr (DIAG) {
                        // per-tile mass of P_hat (codes x scales) and of P
                        if (p.tile_sums != nullptr && valid && j < own_steps) {
                            float sh = 0.0f;
#pragma unroll
                            for (int b = 0; b < 8; ++b) {
                                const uint32_t sf = (sfw[b >> 2] >> (8 * (b & 3))) & 0xFFu;
                                sh = __fmaf_rn(e4m3_to_f32(sf), e2m1x8_sum(code[2 * b]) + e2m1x8_sum(code[2 * b + 1]), sh);
                            }
                            p.tile_sums[out_row * (size_t)p.n_kv_tiles + (kt0 + j)] = make_float2(sh, lsum2.x + lsum2.y);
                        }
                        // copy of this row's P_hat codes and scales
                        if (p.p_codes != nullptr && valid && j < own_steps) {
                            uint4* dc = reinterpret_cast<uint4*>(p.p_codes + out_row * (size_t)(p.Nkv / 2) + n0 / 2);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dc[q] = make_uint4(code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
                            *reinterpret_cast<uint2*>(p.p_sf + out_row * (size_t)(p.Nkv / 16) + n0 / 16) =
                                make_uint2(sfw[0], sfw[1]);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                m_old = m_new;
                mc_old = mc_new;
                if constexpr (BIAS) stage_bias(j + 1);
            }
            // every row's P_hat is in shared memory and its O is rescaled: PV
            if (ok) named_barrier_arrive(id_p, 160); else named_barrier_sync(id_p, 160);
            HIFA4_TRACE_POINT(qt, j, 6);
        }
        // ---------------------------------------------------------- epilogue
        HIFA4_TRACE_POINT(qt, 62, 0);
        if (ok && nt > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_done[qt], (nt - 1) & 1, ctl));
        float l = 0.0f;
        if (ok && nt > 0) {
            tc_fence_after();
            if constexpr (PREORDER) {
                uint32_t lv;
                tmem_ld1(tO + D, lv);
                tmem_wait_ld();
                l = __uint_as_float(lv);
            } else {
                l = l_hp;
            }
        }
        if constexpr (!DEC) {
            if (ok && nt > 0) {
                const float inv = l > 0.0f ? __frcp_rn(l) : 0.0f;
#pragma unroll 1
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + cc, o);
                    tmem_wait_ld_dep(o);
                    float v[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * inv;
                    if (valid) {
                        uint8_t* dst = reinterpret_cast<uint8_t*>(p.o) + (out_row * D + cc) * (OUT == 2 ? 4 : 2);
                        store_out<OUT, 32>(dst, v);
                    }
                }
                if (valid && p.lse != nullptr)
                    p.lse[out_row] = l > 0.0f ? mc_old * 0.69314718055994531f + __logf(l) : -INFINITY;
            }
        } else {
            // merge the four kv ranges of each row. After the first barrier all
            // MMAs of both tiles are done (every thread waited for its tile's
            // last PV), so the K/V ring and the P buffers are free scratch.
            float* part = reinterpret_cast<float*>(smem + C::OFF_K);          // [range][row][MERGE_ROW]
            float2* ml = reinterpret_cast<float2*>(smem + C::OFF_P);          // [range][row] = (mc, l)
            named_barrier_sync(5, 128 * NQT);
            const bool mine = ok && valid && l > 0.0f;
            if (valid) ml[range * 64 + prow] = mine ? make_float2(mc_old, l) : make_float2(0.0f, 0.0f);
            named_barrier_sync(5, 128 * NQT);
            float M = -INFINITY, L = 0.0f;
            if (valid) {
#pragma unroll
                for (int r = 0; r < kDecSplits; ++r) {
                    const float2 e = ml[r * 64 + prow];
                    if (e.y > 0.0f) M = fmaxf(M, e.x);
                }
#pragma unroll
                for (int r = 0; r < kDecSplits; ++r) {
                    const float2 e = ml[r * 64 + prow];
                    if (e.y > 0.0f) L = __fmaf_rn(ex2_approx(e.x - M), e.y, L);
                }
            }
            const float wgt = (mine && L > 0.0f) ? __fdividef(ex2_approx(mc_old - M), L) : 0.0f;
            if (valid) {
                float* dst = part + ((size_t)range * 64 + prow) * C::MERGE_ROW;
#pragma unroll 1
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t o[32];
                    if (mine) {
                        tmem_ld32(tO + cc, o);
                        tmem_wait_ld_dep(o);
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(dst + cc + e) =
                            mine ? make_float4(__uint_as_float(o[e]) * wgt, __uint_as_float(o[e + 1]) * wgt,
                                               __uint_as_float(o[e + 2]) * wgt, __uint_as_float(o[e + 3]) * wgt)
                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
            }
            named_barrier_sync(5, 128 * NQT);
            // thread (range r, row q) writes columns [r*D/4, (r+1)*D/4) of row q
            constexpr int CW = D / kDecSplits;
            if (valid && ok) {
                float v[CW];
#pragma unroll
                for (int e = 0; e < CW; ++e) v[e] = 0.0f;
#pragma unroll
                for (int r = 0; r < kDecSplits; ++r) {
                    const float* src = part + ((size_t)r * 64 + prow) * C::MERGE_ROW + range * CW;
#pragma unroll
                    for (int e = 0; e < CW; e += 4) {
                        const float4 t4 = *reinterpret_cast<const float4*>(src + e);
                        v[e] += t4.x;
                        v[e + 1] += t4.y;
                        v[e + 2] += t4.z;
                        v[e + 3] += t4.w;
                    }
                }
                uint8_t* dst = reinterpret_cast<uint8_t*>(p.o) + (out_row * D + range * CW) * (OUT == 2 ? 4 : 2);
                store_out<OUT, CW>(dst, v);
                if (range == 0 && p.lse != nullptr)
                    p.lse[out_row] = L > 0.0f ? M * 0.69314718055994531f + __logf(L) : -INFINITY;
            }
        }
    }
    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (threadIdx.x == 0) HIFA4_TRACE_POINT(4, 63, 2);
}

template <int D, bool PRE, bool CAUSAL, int OUT, int XT, bool DEC>
static cudaError_t launch_one(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                              cudaStream_t st) {
    using C = Cfg<D, PRE, DEC, XT == 3>;
    auto kern = attn_fwd_kernel<D, PRE, CAUSAL, OUT, XT, DEC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3((unsigned)p.n_work);
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = C::SMEM_BYTES;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, *q, *k, *v, p);
}

template <int D, bool PRE, bool CAUSAL, int OUT, int XT>
static cudaError_t launch_dec(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                              bool dec, cudaStream_t st) {
    if constexpr (D <= 128) {
        if (dec) return launch_one<D, PRE, CAUSAL, OUT, XT, true>(q, k, v, p, st);
    } else {
        if (dec) return cudaErrorInvalidValue;
    }
    return launch_one<D, PRE, CAUSAL, OUT, XT, false>(q, k, v, p, st);
}

template <int D, bool PRE, bool CAUSAL, int OUT>
static cudaError_t launch_extras(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v,
                                 const AttnParams& p, int xt, bool dec, cudaStream_t st) {
    switch (xt) {
        case 0: return launch_dec<D, PRE, CAUSAL, OUT, 0>(q, k, v, p, dec, st);
        case 1: return launch_dec<D, PRE, CAUSAL, OUT, 1>(q, k, v, p, dec, st);
        case 2: return launch_dec<D, PRE, CAUSAL, OUT, 2>(q, k, v, p, dec, st);
        default:
            if constexpr (D == 128) {
                if (!dec) return launch_one<D, PRE, CAUSAL, OUT, 3, false>(q, k, v, p, st);
            }
            return cudaErrorInvalidValue;
    }
}

template <int D, bool PRE, bool CAUSAL>
static cudaError_t launch_out(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                              int out, int xt, bool dec, cudaStream_t st) {
    switch (out) {
        case 0: return launch_extras<D, PRE, CAUSAL, 0>(q, k, v, p, xt, dec, st);
        case 1: return launch_extras<D, PRE, CAUSAL, 1>(q, k, v, p, xt, dec, st);
        default: return launch_extras<D, PRE, CAUSAL, 2>(q, k, v, p, xt, dec, st);
    }
}

template <int D>
static cudaError_t launch_d(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                            int norm, bool causal, int out, int xt, bool dec, cudaStream_t st) {
    if (norm == 0)
        return causal ? launch_out<D, true, true>(q, k, v, p, out, xt, dec, st)
                      : launch_out<D, true, false>(q, k, v, p, out, xt, dec, st);
    return causal ? launch_out<D, false, true>(q, k, v, p, out, xt, dec, st)
                  : launch_out<D, false, false>(q, k, v, p, out, xt, dec, st);
}

cudaError_t launch_attention(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const AttnParams& p, int D, int norm, bool causal, int out_dtype, int xt, bool dec,
                             cudaStream_t st) {
    switch (D) {
        case 64: return launch_d<64>(tmQ, tmK, tmV, p, norm, causal, out_dtype, xt, dec, st);
        case 128: return launch_d<128>(tmQ, tmK, tmV, p, norm, causal, out_dtype, xt, dec, st);
        case 256: return launch_d<256>(tmQ, tmK, tmV, p, norm, causal, out_dtype, xt, dec, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hifa4
