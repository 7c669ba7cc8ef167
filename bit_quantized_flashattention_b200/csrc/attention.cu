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
//   warp 0      TMA / bulk-copy producer: Q_hat tiles once, then K_hat and
//               V_hat^T tiles (128 keys) with their scale atoms, 3-stage rings
//   warp 1      TMEM owner; moves the Q scales to TMEM and issues every S MMA
//   warps 2, 3  PV MMA issuers, one per query tile
//   warps 4..   one softmax warpgroup per query tile, thread t owns row t:
//               block maxima of S, running max, P = 2^(S*c - RN(m*c)),
//               P quantized per 16 keys to E2M1 + E4M3 in registers, O rescaled
//               in TMEM when some row's max moved, P_hat codes and scales
//               written to shared memory for the PV MMA.
// The S MMAs run one at a time through one 128-column S buffer in TMEM, in the
// order (kv tile 0, query tile 0), (0, 1), (1, 0), ...: once a warpgroup has
// loaded its scores it arrives (without waiting) at its named barrier
// "scores loaded", and the S issuer, blocked in that barrier, issues the next S
// MMA of the order; no warp polls an mbarrier on this path. After the second
// named barrier of the tile (P_hat stored, O rescaled) the tile's PV issuer
// issues its PV MMA. An MMA depends only on tcgen05 operations already observed
// complete through an mbarrier, or issued earlier by the same thread.
// With P-Reordering the V tile carries 16 extra rows: a row of E2M1 ones
// (scale 1.0) and 15 zero rows, so the PV MMA also produces sum(P_hat) in
// output column D: the normalizer from exactly the codes x scales the MMA used.
// TMEM (512 columns): S [0,128), O tiles [128, 128 + NQT*NO), NO = D (+16),
// then the scale-factor regions of Q, K, P and V (P and V per query tile).
// Every mbarrier wait is bounded; when one gives up the CTA records
// HIFA4_ERR_TIMEOUT in the workspace, drains its copies and MMAs, frees TMEM
// and exits. The named barriers also OR a failure flag over their threads, so a
// warpgroup and its issuer leave the loop together.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hifa4_device.cuh"
#include "hifa4_kernels.h"

namespace hifa4 {

constexpr int kStages = 4;
constexpr int kSmWarp0 = 4;          // first softmax warp (0: loads, 1: TMEM owner + S MMAs, 2-3: PV MMAs)

template <int D, bool PREORDER>
struct Cfg {
    static constexpr int NQT = D == 256 ? 1 : 2;          // 128-row query tiles per CTA
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
    static constexpr int SFP_BYTES = 2 * 512;
    static constexpr int NO = PREORDER ? D + 16 : D;      // accumulator columns per query tile
    static constexpr int NCH = D / 32;                    // 32-column chunks of O
    // TMEM columns
    static constexpr uint32_t COL_S = 0;
    static constexpr uint32_t COL_O = 128;                                // + qt * NO
    static constexpr uint32_t COL_SFQ = COL_O + NQT * NO;                 // + qt * 4 * KS
    static constexpr uint32_t COL_SFK = COL_SFQ + NQT * 4 * KS;
    static constexpr uint32_t COL_SFP = COL_SFK + 4 * KS;                 // + qt * 8
    static constexpr uint32_t COL_SFV = COL_SFP + NQT * 8;                 // + qt * 2 * SFV_PER_KS
    // scale columns per PV K step: one 4-column block per 128 rows of the B operand
    static constexpr int SFV_PER_KS = 4 * (NRB + ((PREORDER && D >= 128) ? 1 : 0));
    static constexpr uint32_t COL_END = COL_SFV + NQT * 2 * SFV_PER_KS;
    static_assert(COL_END <= 512, "TMEM budget");
    // shared memory offsets (operand tiles 1024-aligned)
    static constexpr int OFF_Q = 0;                                       // + qt * Q_BYTES
    static constexpr int OFF_K = OFF_Q + NQT * Q_BYTES;
    static constexpr int OFF_V = OFF_K + kStages * K_BYTES;
    static constexpr int OFF_P = OFF_V + kStages * V_STRIDE;              // + (qt * 2 + buf) * P_BYTES
    static constexpr int OFF_SFQ = OFF_P + NQT * 2 * P_BYTES;             // + qt * SFQK_BYTES
    static constexpr int OFF_SFK = OFF_SFQ + NQT * SFQK_BYTES;
    static constexpr int OFF_SFV = OFF_SFK + kStages * SFQK_BYTES;
    static constexpr int OFF_SFP = OFF_SFV + kStages * SFV_BYTES;         // + (qt * 2 + buf) * SFP_BYTES
    static constexpr int OFF_ONES = OFF_SFP + NQT * 2 * SFP_BYTES;
    static constexpr int OFF_LUT = OFF_ONES + 512;                        // float [128]
    static constexpr int OFF_BAR = OFF_LUT + 128 * 4;
    static constexpr int OFF_MISC = OFF_BAR + 256;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;              // + alignment slack
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages];
    uint64_t v_full[kStages];
    uint64_t v_empty[kStages][2];   // K and V slot no longer read by query tile x's MMAs
    uint64_t s_full[2];             // S of query tile x is in TMEM
    uint64_t o_done[2];             // PV MMA of query tile x finished
    uint64_t sfk_full;              // K scales of the next kv tile moved to TMEM
    uint64_t drain[3];              // teardown: MMAs issued by the starter / by each tile's leader
};
static_assert(sizeof(Bars) <= 256, "barrier area");

#ifndef HIFA4_TRACE_POINT
#define HIFA4_TRACE_POINT(role, j, e)
#endif

__device__ __forceinline__ uint32_t p_swizzle64(uint32_t row, uint32_t chunk) {
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

template <int OUT>
__device__ __forceinline__ void store_out32(void* dst, const float (&v)[32]) {
    if constexpr (OUT == 2) {
        float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
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
        for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
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

template <int D, bool PREORDER, bool CAUSAL, int OUT, bool DUMP>
__global__ void __launch_bounds__(Cfg<D, PREORDER>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = Cfg<D, PREORDER>;
    constexpr int NQT = C::NQT;
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
    // One work unit = up to NQT consecutive 128-row query tiles of one group.
    const int w = blockIdx.x;
    const int units_per_grp = (p.Tq + NQT - 1) / NQT;
    int grp, t0;
    if (p.heavy_first) {
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
    const int n_qt = min(NQT, p.Tq - t0);
    const int rows_in_grp = p.G * p.Nq;
    // kv tiles each query tile visits (causal: up to the last visible key of its last row)
    auto kv_tiles_of = [&](int qt) -> int {
        if (qt >= n_qt) return 0;
        if (!CAUSAL) return p.n_kv_tiles;
        const int p0 = (t0 + qt) * 128;
        const int p_max = min(p0 + 127, rows_in_grp - 1);
        const int i_max = (p_max / p.Nq == p0 / p.Nq) ? (p_max % p.Nq) : (p.Nq - 1);
        return min(p.n_kv_tiles, (i_max + p.Nkv - p.Nq) / 128 + 1);
    };
    int n_tiles[2];
    n_tiles[0] = kv_tiles_of(0);
    n_tiles[1] = NQT > 1 ? kv_tiles_of(1) : 0;
    const int n_tiles_max = max(n_tiles[0], n_tiles[1]);

    // The S MMAs run one at a time through the one S buffer, in the order
    // (kv tile 0, query tile 0), (0, 1), (1, 0), (1, 1), ... skipping the kv
    // tiles a query tile does not visit. The item after (j, x) in that order:
    auto next_item = [&](int j, int x, int& nj, int& nx) -> bool {
#pragma unroll 1
        for (int guard = 0; guard < 2 * NQT + 2; ++guard) {
            if (++x >= NQT) { x = 0; ++j; }
            if (j >= n_tiles_max) return false;
            if (j < n_tiles[x]) { nj = j; nx = x; return true; }
        }
        return false;
    };

    // --------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            for (int x = 0; x < 2; ++x) mbar_init(&bars->v_empty[s][x], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->o_done[x], 1);
        }
        for (int k = 0; k < 3; ++k) mbar_init(&bars->drain[k], 1);
        mbar_init(&bars->sfk_full, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x >= 128 && threadIdx.x < 256) {
        const uint32_t i = threadIdx.x - 128;
        lut[i] = (i == 0) ? 0.0f : __frcp_rn(e4m3_to_f32(i));
        // normalizer block of V^T (rows D..D+15 of every stage): one row of E2M1
        // ones (code 2 in both nibbles), 15 zero rows; and the scale atom of the
        // ones row (row 0 of an atom = 1.0) used when D >= 128.
        for (int s = 0; s < kStages; ++s) {
            uint32_t* row = reinterpret_cast<uint32_t*>(smem + C::OFF_V + s * C::V_STRIDE + D * 64);
            for (int k = i; k < 16 * 16; k += 128) row[k] = (k < 16) ? 0x22222222u : 0u;
        }
        reinterpret_cast<uint32_t*>(smem + C::OFF_ONES)[i] = (i == 0) ? 0x38383838u : 0u;
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

    // Scale atoms moved shared->TMEM, and the MMAs. Issued by one thread at a
    // time; an MMA is issued only after every tcgen05 operation it depends on
    // has completed (observed through an mbarrier), except where one thread
    // issues both: its tcgen05 operations run in issue order.
    // Shared-memory descriptors: a base descriptor plus (byte offset >> 4) in
    // the 14-bit address field (all shared addresses are below 256 KB).
    const uint32_t idesc_s = idesc_fp4_block16(128);
    auto sf_desc = [&](uint32_t off) { return smem_desc(sbase + off, 0u, 128u, 0u); };
    const uint64_t qk_desc0 = smem_desc(sbase, 16u, C::QK_SBO, C::QK_SWZ);
    const uint64_t pv_desc0 = smem_desc(sbase, 16u, 512u, 4u);
    // first and last query tile (in S order) that visit kv tile j
    auto first_x_of = [&](int j) -> int { return j < n_tiles[0] ? 0 : 1; };
    auto last_x_of = [&](int j) -> int { return (NQT > 1 && j < n_tiles[1]) ? 1 : 0; };
    auto copy_sfk = [&](int j) {
        const int st = j % kStages;
#pragma unroll
        for (int s = 0; s < C::KS; ++s)
            tmem_cp_scale_atom(tmem + C::COL_SFK + 4 * s, sf_desc(C::OFF_SFK + st * C::SFQK_BYTES + 512 * s));
    };
    auto copy_sfv = [&](int j, int x) {
        const int st = j % kStages;
        const uint32_t sfv = C::OFF_SFV + st * C::SFV_BYTES;
        const uint32_t col_sfv = C::COL_SFV + x * 2 * C::SFV_PER_KS;
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int rb = 0; rb < C::NRB; ++rb)
                tmem_cp_scale_atom(tmem + col_sfv + s * C::SFV_PER_KS + 4 * rb, sf_desc(sfv + (rb * 2 + s) * 512));
    };
    // S = Q_hat(x) K_hat(j)^T. The issuer of the last S MMA on tile j then
    // moves the next tile's K scales in (they replace tile j's only after that
    // MMA: same thread, issue order) and signals sfk_full; the first S MMA on a
    // tile waits for that signal (the scales of tile 0 come with the first MMA).
    // Returns false if a wait gave up.
    auto issue_s = [&](int j, int x) -> bool {
        const int st = j % kStages;
        if (j > 0 && x == first_x_of(j) && !mbar_wait_poll(&bars->sfk_full, (j - 1) & 1, ctl, 32)) {
            tc_commit(&bars->s_full[x]);
            return false;
        }
        tc_fence_after();
        const uint64_t kd = qk_desc0 + ((C::OFF_K + st * C::K_BYTES) >> 4);
        const uint64_t qd = qk_desc0 + ((C::OFF_Q + x * C::Q_BYTES) >> 4);
#pragma unroll
        for (int s = 0; s < C::KS; ++s)
            mma_fp4_block16(tmem + C::COL_S, qd + 2 * s, kd + 2 * s, idesc_s, tmem + C::COL_SFQ + x * 4 * C::KS + 4 * s,
                            tmem + C::COL_SFK + 4 * s, s > 0 ? 1u : 0u);
        tc_commit(&bars->s_full[x]);
        if (x == last_x_of(j) && j + 1 < n_tiles_max) {
            if (!mbar_wait_poll(&bars->k_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, ctl, 32)) return false;
            copy_sfk(j + 1);
            tc_commit(&bars->sfk_full);
        }
        return true;
    };
    // O(x) += P_hat(x, j) V_hat(j) (P scales written to TMEM by the softmax
    // threads, V scales of tile j already in x's columns); then the V scales
    // of tile j + 1 are moved in for the next PV MMA of this tile.
    auto issue_pv = [&](int j, int x) -> bool {
        const int st = j % kStages;
        const uint64_t vd = pv_desc0 + ((C::OFF_V + st * C::V_STRIDE) >> 4);
        const uint64_t pd = pv_desc0 + ((C::OFF_P + (x * 2 + (j & 1)) * C::P_BYTES) >> 4);
        const uint32_t col_sfv = C::COL_SFV + x * 2 * C::SFV_PER_KS;
        const uint32_t o = tmem + C::COL_O + x * C::NO;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const uint32_t acc = (j > 0 || s > 0) ? 1u : 0u;
            const uint32_t sfa = tmem + C::COL_SFP + x * 8 + 4 * s;
            const uint32_t sfb = tmem + col_sfv + s * C::SFV_PER_KS;
            if constexpr (D == 256 && PREORDER) {
                mma_fp4_block16(o, pd + 2 * s, vd + 2 * s, idesc_fp4_block16(128), sfa, sfb, acc);
                mma_fp4_block16(o + 128, pd + 2 * s, vd + ((128 * 64) >> 4) + 2 * s, idesc_fp4_block16(144), sfa,
                                sfb + 4, acc);
            } else {
                mma_fp4_block16(o, pd + 2 * s, vd + 2 * s, idesc_fp4_block16(C::NO), sfa, sfb, acc);
            }
        }
        tc_commit(&bars->o_done[x]);
        tc_commit(&bars->v_empty[st][x]);
        if (j + 1 < n_tiles[x]) {
            if (!mbar_wait_poll(&bars->v_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, ctl, 32)) return false;
            copy_sfv(j + 1, x);
        }
        return true;
    };

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // The set-up above overlaps the end of the previous kernel in the
        // stream (programmatic dependent launch); the packed operands are read
        // only after it has completed. Every other read of those operands
        // goes through this warp's copies. A slot is refilled once every query
        // tile that read the previous kv tile in it has released it.
        grid_dependency_wait();
        if (lane == 0 && !p.stall_loads) {
            int issued = 0;
            bool ok = true;
            mbar_arrive_expect_tx(&bars->q_full, n_qt * (C::Q_BYTES + C::SFQK_BYTES));
            for (int qt = 0; qt < n_qt; ++qt) {
                tma_load_2d(smem + C::OFF_Q + qt * C::Q_BYTES, &tmQ, 0, grp * rows_in_grp + (t0 + qt) * 128,
                            &bars->q_full);
                bulk_load(smem + C::OFF_SFQ + qt * C::SFQK_BYTES,
                          p.qs + ((size_t)grp * p.Tq + t0 + qt) * C::SFQK_BYTES, C::SFQK_BYTES, &bars->q_full);
            }
            for (int j = 0; j < n_tiles_max && ok; ++j) {
                const int st = j % kStages;
                const int jp = j - kStages;                          // previous kv tile in this slot
                const uint32_t ph = (jp / kStages) & 1;
                // a finished PV MMA of tile jp also means its S MMAs finished
                for (int x = 0; x < NQT && jp >= 0 && ok; ++x)
                    if (jp < n_tiles[x] && !mbar_wait_poll(&bars->v_empty[st][x], ph, ctl, 256)) ok = false;
                if (!ok) break;
                mbar_arrive_expect_tx(&bars->k_full[st], C::K_BYTES + C::SFQK_BYTES);
                tma_load_2d(smem + C::OFF_K + st * C::K_BYTES, &tmK, 0, grp * p.Nkv + j * 128, &bars->k_full[st]);
                bulk_load(smem + C::OFF_SFK + st * C::SFQK_BYTES,
                          p.ks + ((size_t)grp * p.n_kv_tiles + j) * C::SFQK_BYTES, C::SFQK_BYTES, &bars->k_full[st]);
                issued = 2 * j + 1;
                mbar_arrive_expect_tx(&bars->v_full[st], C::V_TMA_BYTES + C::SFV_BYTES);
                tma_load_2d(smem + C::OFF_V + st * C::V_STRIDE, &tmV, j * 64, grp * D, &bars->v_full[st]);
                bulk_load(smem + C::OFF_SFV + st * C::SFV_BYTES,
                          p.vts + ((size_t)grp * p.n_kv_tiles + j) * C::SFV_BYTES, C::SFV_BYTES, &bars->v_full[st]);
                issued = 2 * j + 2;
            }
            if (!ok) {
                // drain the copies still in flight before the CTA exits
                const int nk = (issued + 1) / 2, nv = issued / 2;
                for (int j = max(0, nk - kStages); j < nk; ++j)
                    mbar_wait_drain(&bars->k_full[j % kStages], (j / kStages) & 1, p.wait_limit_ns);
                for (int j = max(0, nv - kStages); j < nv; ++j)
                    mbar_wait_drain(&bars->v_full[j % kStages], (j / kStages) & 1, p.wait_limit_ns);
                mbar_wait_drain(&bars->q_full, 0, p.wait_limit_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- S issuer
        // Moves the Q scales (and the first tiles' K and V scales) to TMEM,
        // issues the first S MMA, then walks the S order: once the consumer of
        // an S tile has loaded it (named barrier "scores loaded" of that
        // warpgroup, which arrives without waiting) the next S MMA is issued.
        // A warp blocked in a named barrier takes no issue slots.
        bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->q_full, 0, ctl));
        int j = 0, x = 0;
        bool more = next_item(0, -1, j, x);
        if (ok && more) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->k_full[0], 0, ctl));
        if (ok && more) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->v_full[0], 0, ctl));
        bool issued_any = false;
        if (ok) {
            tc_fence_after();
            if (lane == 0) {
                for (int qt = 0; qt < n_qt; ++qt) {
#pragma unroll
                    for (int s = 0; s < C::KS; ++s)
                        tmem_cp_scale_atom(tmem + C::COL_SFQ + qt * 4 * C::KS + 4 * s,
                                           sf_desc(C::OFF_SFQ + qt * C::SFQK_BYTES + 512 * s));
                    // scale atom of the normalizer rows (rows D.. of the V operand)
                    if constexpr (PREORDER && D >= 128) {
#pragma unroll
                        for (int s = 0; s < 2; ++s)
                            tmem_cp_scale_atom(tmem + C::COL_SFV + qt * 2 * C::SFV_PER_KS + s * C::SFV_PER_KS + 4 * C::NRB,
                                               sf_desc(C::OFF_ONES));
                    }
                }
                if (more) {
                    copy_sfk(0);
                    for (int qt = 0; qt < n_qt; ++qt) copy_sfv(0, qt);
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
        // the warpgroup arrives on every kv tile, also after a failure
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
        const int prow = (t0 + qt) * 128 + row;
        const bool valid = qt < n_qt && prow < rows_in_grp;
        const int qi = prow % p.Nq;
        const int last = valid ? (CAUSAL ? qi + p.Nkv - p.Nq : p.Nkv - 1) : -1;
        const size_t out_row = (size_t)grp * rows_in_grp + prow;
        const int nt = n_tiles[qt];
        const float c = p.c;
        const float2 c2 = make_float2(c, c);
        const float one_sixth = rn_one_sixth();
        const uint32_t lut_s = smem_u32(lut);
        float m_old = -INFINITY, mc_old = 0.0f, l_hp = 0.0f;
        bool ok = true;                                     // false once a wait gave up (then no more work)
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
            // warpgroup cannot reach the next tile's arrival before the issuer
            // has passed this barrier: that S MMA is issued after it); after a
            // failure the waits no longer hold it back, so it syncs instead.
            if (ok) named_barrier_arrive(id_s, 160); else named_barrier_sync(id_s, 160);
            HIFA4_TRACE_POINT(qt, j, 2);
            if (ok) {
                const int n0 = j * 128;
                if (n0 + 127 > last) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        if (n0 + 2 * e > last) S[e].x = -INFINITY;
                        if (n0 + 2 * e + 1 > last) S[e].y = -INFINITY;
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
                // P = 2^(S*c - mc), 8 blocks of 16 keys to E2M1 codes + E4M3 scales
                uint32_t code[16];
                uint32_t sfw[2] = {0u, 0u};
                float2 lsum2 = make_float2(0.0f, 0.0f);
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
                            const float2 t = __ffma2_rn(S[8 * b + 4 * h + e], c2, nmc2);
                            const float2 P = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                            if constexpr (!PREORDER) lsum2 = __fadd2_rn(lsum2, P);
                            const float2 yy = __fmul2_rn(P, r2);
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
                    const uint32_t pb = sbase + C::OFF_P + (qt * 2 + (j & 1)) * C::P_BYTES;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        sts_v4(pb + p_swizzle64(row, q), code[4 * q], code[4 * q + 1], code[4 * q + 2], code[4 * q + 3]);
                    // the row's E4M3 scales straight into the TMEM column the PV MMA
                    // reads for it (row r: lane r, column base + r/32 of each K step;
                    // the previous PV, the last reader, is done)
                    tmem_st1(tl + C::COL_SFP + qt * 8 + wq, sfw[0]);
                    tmem_st1(tl + C::COL_SFP + qt * 8 + 4 + wq, sfw[1]);
                    tmem_wait_st();
                    if constexpr (DUMP) {
                        // debug copy of this row's P_hat codes and scales
                        if (valid) {
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
            }
            // every row's P_hat is in shared memory and its O is rescaled: PV
            if (ok) named_barrier_arrive(id_p, 160); else named_barrier_sync(id_p, 160);
            HIFA4_TRACE_POINT(qt, j, 6);
        }
        // ---------------------------------------------------------- epilogue
        if (ok && nt > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_done[qt], (nt - 1) & 1, ctl));
        if (ok && nt > 0) {
            tc_fence_after();
            float l;
            if constexpr (PREORDER) {
                uint32_t lv;
                tmem_ld1(tO + D, lv);
                tmem_wait_ld();
                l = __uint_as_float(lv);
            } else {
                l = l_hp;
            }
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
                    store_out32<OUT>(dst, v);
                }
            }
            if (valid && p.lse != nullptr)
                p.lse[out_row] = l > 0.0f ? mc_old * 0.69314718055994531f + __logf(l) : -INFINITY;
        }
    }
    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool PRE, bool CAUSAL, int OUT, bool DUMP>
static cudaError_t launch_one(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                              cudaStream_t st) {
    using C = Cfg<D, PRE>;
    auto kern = attn_fwd_kernel<D, PRE, CAUSAL, OUT, DUMP>;
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

template <int D, bool PRE, bool CAUSAL, int OUT>
static cudaError_t launch_dump(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                               bool dump, cudaStream_t st) {
    return dump ? launch_one<D, PRE, CAUSAL, OUT, true>(q, k, v, p, st)
                : launch_one<D, PRE, CAUSAL, OUT, false>(q, k, v, p, st);
}

template <int D, bool PRE, bool CAUSAL>
static cudaError_t launch_out(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                              int out, bool dump, cudaStream_t st) {
    switch (out) {
        case 0: return launch_dump<D, PRE, CAUSAL, 0>(q, k, v, p, dump, st);
        case 1: return launch_dump<D, PRE, CAUSAL, 1>(q, k, v, p, dump, st);
        default: return launch_dump<D, PRE, CAUSAL, 2>(q, k, v, p, dump, st);
    }
}

template <int D>
static cudaError_t launch_d(const CUtensorMap* q, const CUtensorMap* k, const CUtensorMap* v, const AttnParams& p,
                            int norm, bool causal, int out, bool dump, cudaStream_t st) {
    if (norm == 0)
        return causal ? launch_out<D, true, true>(q, k, v, p, out, dump, st)
                      : launch_out<D, true, false>(q, k, v, p, out, dump, st);
    return causal ? launch_out<D, false, true>(q, k, v, p, out, dump, st)
                  : launch_out<D, false, false>(q, k, v, p, out, dump, st);
}

cudaError_t launch_attention(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const AttnParams& p, int D, int norm, bool causal, int out_dtype, bool dump,
                             cudaStream_t st) {
    switch (D) {
        case 64: return launch_d<64>(tmQ, tmK, tmV, p, norm, causal, out_dtype, dump, st);
        case 128: return launch_d<128>(tmQ, tmK, tmV, p, norm, causal, out_dtype, dump, st);
        case 256: return launch_d<256>(tmQ, tmK, tmV, p, norm, causal, out_dtype, dump, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hifa4
