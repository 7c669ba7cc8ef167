// C ABI of the 4-bit attention library (declared in include/hifa4.h):
// argument validation, TMA tensor maps and kernel launches. No allocation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/hifa4.h"
#include "api_internal.h"
#include "hifa4_kernels.h"

using namespace hifa4;

namespace {

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;   // 2 s
std::atomic<long long> g_wait_limit_ns{0};

unsigned long long wait_limit_ns() {
    const long long lim = g_wait_limit_ns.load();
    return lim > 0 ? (unsigned long long)lim : kDefaultWaitNs;
}
std::atomic<int> g_stall_loads{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(int B, int Hq, int Hkv, int Nq, int Nkv, int D) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0) return false;
    if (Hq % Hkv != 0) return false;
    if (D != 64 && D != 128 && D != 256) return false;
    if (Nkv % 128 != 0 || Nq % 16 != 0) return false;
    return true;
}

struct Sizes {
    size_t qc, qs, kc, ks, vtc, vts;
    int Tq;
};

Sizes sizes_of(int B, int Hq, int Hkv, int Nq, int Nkv, int D) {
    Sizes s{};
    const int G = Hq / Hkv;
    s.Tq = (G * Nq + 127) / 128;
    const size_t KS = (size_t)D / 64;
    const size_t NRB = ((size_t)D + 127) / 128;
    s.qc = (size_t)B * Hq * Nq * (D / 2);
    s.qs = (size_t)B * Hkv * s.Tq * KS * 512;
    s.kc = (size_t)B * Hkv * Nkv * (D / 2);
    s.ks = (size_t)B * Hkv * (Nkv / 128) * KS * 512;
    s.vtc = (size_t)B * Hkv * D * (Nkv / 2);
    s.vts = (size_t)B * Hkv * (Nkv / 128) * NRB * 2 * 512;
    return s;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D u8 tensor map: `rows` rows of `row_bytes` bytes, box of box_rows x row_bytes... (inner box = box_x bytes).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_x, uint32_t box_y,
              CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner_bytes, rows};
    cuuint64_t strides[1] = {inner_bytes};
    cuuint32_t box[2] = {box_x, box_y};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// The kernels' split-kv decode mode applies: asked for, D <= 128, a group's
// query rows fit in half a tile, and every one of the kv ranges gets a tile.
bool decode_mode(int Hq, int Hkv, int Nq, int Nkv, int D, unsigned flags) {
    return (flags & HIFA4_SPLIT_KV) != 0 && D <= 128 && (long long)(Hq / Hkv) * Nq <= 64 &&
           Nkv / 128 >= kDecodeSplits;
}

// Checks of the optional steps before quantization; want_q / want_k: the
// call quantizes Q / K (their positions are then needed with RoPE).
hifa4_status check_prequant(const hifa4_prequant& x, bool want_q, bool want_k) {
    if ((x.s == nullptr) != (x.s_inv == nullptr)) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(x.s) || !aligned16(x.s_inv)) return HIFA4_ERR_INVALID_ARG;
    if ((x.rope_cos == nullptr) != (x.rope_sin == nullptr)) return HIFA4_ERR_INVALID_ARG;
    if (x.rope_cos != nullptr) {
        if (!aligned16(x.rope_cos) || !aligned16(x.rope_sin) || x.n_pos <= 0) return HIFA4_ERR_INVALID_ARG;
        if (want_q && (x.q_pos == nullptr || (reinterpret_cast<uintptr_t>(x.q_pos) & 3u))) return HIFA4_ERR_INVALID_ARG;
        if (want_k && (x.k_pos == nullptr || (reinterpret_cast<uintptr_t>(x.k_pos) & 3u))) return HIFA4_ERR_INVALID_ARG;
    }
    if ((x.q_mean == nullptr) != (x.s_bias == nullptr)) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(x.q_mean) || !aligned16(x.s_bias)) return HIFA4_ERR_INVALID_ARG;
    return HIFA4_OK;
}

void set_prequant(QuantArgs& a, const hifa4_prequant& x) {
    a.s = x.s;
    a.s_inv = x.s_inv;
    a.rope_cos = x.rope_cos;
    a.rope_sin = x.rope_sin;
    a.q_pos = x.q_pos;
    a.k_pos = x.k_pos;
    a.n_pos = x.n_pos;
    a.q_mean = x.q_mean;
    a.s_bias = x.s_bias;
}

}  // namespace

hifa4_status hifa4::from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return HIFA4_OK;
    g_last_cuda_error = e;
    return HIFA4_ERR_CUDA;
}

hifa4_status hifa4::check_attention_args(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                         float sm_scale, unsigned flags, hifa4_norm_mode norm, const void* o,
                                         hifa4_dtype o_dtype, const float* lse) {
    if (in == nullptr || o == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (!shape_ok(B, Hq, Hkv, Nq, Nkv, D)) return HIFA4_ERR_UNSUPPORTED;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return HIFA4_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)(HIFA4_CAUSAL | HIFA4_SPLIT_KV)) != 0) return HIFA4_ERR_INVALID_ARG;
    if ((flags & HIFA4_CAUSAL) != 0 && Nq > Nkv) return HIFA4_ERR_UNSUPPORTED;
    if (norm != HIFA4_NORM_P_REORDER && norm != HIFA4_NORM_HIGH_PRECISION_L) return HIFA4_ERR_INVALID_ARG;
    if (o_dtype != HIFA4_F16 && o_dtype != HIFA4_BF16 && o_dtype != HIFA4_F32) return HIFA4_ERR_INVALID_ARG;
    const void* ptrs[6] = {in->qc, in->qs, in->kc, in->ks, in->vtc, in->vts};
    for (const void* q : ptrs)
        if (q == nullptr || !aligned16(q)) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(o) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u))) return HIFA4_ERR_INVALID_ARG;
    const long long rows_q = (long long)B * Hq * Nq, rows_k = (long long)B * Hkv * Nkv, rows_v = (long long)B * Hkv * D;
    if (rows_q > INT32_MAX || rows_k > INT32_MAX || rows_v * (Nkv / 128) > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    const Sizes sz = sizes_of(B, Hq, Hkv, Nq, Nkv, D);
    const int nqt = D == 256 ? 1 : 2;              // query tiles per CTA (see attention.cu)
    if ((long long)B * Hkv * ((sz.Tq + nqt - 1) / nqt) > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    return HIFA4_OK;
}

namespace {

hifa4_status attention_impl(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D, float sm_scale,
                            unsigned flags, hifa4_norm_mode norm, void* o, hifa4_dtype o_dtype, float* lse,
                            const hifa4_attention_extras* ex, void* workspace, hifa4_stream_t stream) {
    const hifa4_status chk = check_attention_args(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse);
    if (chk != HIFA4_OK) return chk;
    if (workspace == nullptr || !aligned16(workspace)) return HIFA4_ERR_INVALID_ARG;
    hifa4_attention_extras x{};
    if (ex != nullptr) x = *ex;
    if ((x.p_codes == nullptr) != (x.p_scales == nullptr)) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(x.p_codes) || !aligned16(x.p_scales) || !aligned16(x.s_bias) || !aligned16(x.tile_sums))
        return HIFA4_ERR_INVALID_ARG;
    const int xt = (x.p_codes != nullptr || x.tile_sums != nullptr) ? 2 : (x.s_bias != nullptr ? 1 : 0);
    const bool causal = (flags & HIFA4_CAUSAL) != 0;
    const long long rows_q = (long long)B * Hq * Nq, rows_k = (long long)B * Hkv * Nkv, rows_v = (long long)B * Hkv * D;
    const Sizes sz = sizes_of(B, Hq, Hkv, Nq, Nkv, D);
    const int nqt = D == 256 ? 1 : 2;              // query tiles per CTA (see attention.cu)
    const bool dec = decode_mode(Hq, Hkv, Nq, Nkv, D, flags);
    const long long n_work = (long long)B * Hkv * (dec ? 1 : (sz.Tq + nqt - 1) / nqt);

    const CUtensorMapSwizzle swz_qk =
        D == 64 ? CU_TENSOR_MAP_SWIZZLE_32B : (D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, in->qc, (uint64_t)D / 2, (uint64_t)rows_q, D / 2, 128, swz_qk) ||
        !make_map(&tk, in->kc, (uint64_t)D / 2, (uint64_t)rows_k, D / 2, 128, swz_qk) ||
        !make_map(&tv, in->vtc, 64, (uint64_t)rows_v * (Nkv / 128), 64, (uint32_t)D, CU_TENSOR_MAP_SWIZZLE_64B))
        return from_cuda(cudaErrorInvalidValue);

    AttnParams p{};
    p.qs = static_cast<const uint8_t*>(in->qs);
    p.ks = static_cast<const uint8_t*>(in->ks);
    p.vts = static_cast<const uint8_t*>(in->vts);
    p.o = o;
    p.lse = lse;
    p.s_bias = x.s_bias;
    p.p_codes = x.p_codes;
    p.p_sf = x.p_scales;
    p.tile_sums = reinterpret_cast<float2*>(x.tile_sums);
    p.status = static_cast<uint32_t*>(workspace);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.G = Hq / Hkv;
    p.Tq = sz.Tq;
    p.n_kv_tiles = Nkv / 128;
    p.n_work = (int)n_work;
    p.heavy_first = (!dec && causal && Nq % (128 * nqt) == 0) ? 1 : 0;
    p.c = (float)((double)sm_scale * 1.4426950408889634074);
    p.wait_limit_ns = wait_limit_ns();
    p.stall_loads = g_stall_loads.load();
    const int out = o_dtype == HIFA4_F16 ? 0 : (o_dtype == HIFA4_BF16 ? 1 : 2);
    return from_cuda(launch_attention(&tq, &tk, &tv, p, D, (int)norm, causal, out, xt, dec,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

size_t hifa4_packed_bytes(int B, int Hq, int Hkv, int Nq, int Nkv, int D, size_t out[6]) {
    if (!shape_ok(B, Hq, Hkv, Nq, Nkv, D)) return 0;
    const Sizes s = sizes_of(B, Hq, Hkv, Nq, Nkv, D);
    if (out != nullptr) {
        out[0] = s.qc;
        out[1] = s.qs;
        out[2] = s.kc;
        out[3] = s.ks;
        out[4] = s.vtc;
        out[5] = s.vts;
    }
    return s.qc + s.qs + s.kc + s.ks + s.vtc + s.vts;
}

int hifa4_attention_splits(int B, int Hq, int Hkv, int Nq, int Nkv, int D, unsigned flags) {
    if (!shape_ok(B, Hq, Hkv, Nq, Nkv, D)) return 0;
    return decode_mode(Hq, Hkv, Nq, Nkv, D, flags) ? kDecodeSplits : 1;
}

size_t hifa4_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nkv, int D) {
    (void)B; (void)Hq; (void)Hkv; (void)Nq; (void)Nkv; (void)D;
    return 256;                                    // the status word, padded to 256 bytes
}

hifa4_status hifa4_calibrate_smooth(const void* q, const void* k, hifa4_dtype dtype, int B, int Hq, int Hkv, int N,
                                    int D, float alpha, float* s, float* s_inv, hifa4_stream_t stream) {
    if (q == nullptr || k == nullptr || s == nullptr || s_inv == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (dtype != HIFA4_F16 && dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || Hq % Hkv != 0) return HIFA4_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return HIFA4_ERR_UNSUPPORTED;
    if (!(alpha > 0.0f && alpha <= 1.0f)) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(s) || !aligned16(s_inv)) return HIFA4_ERR_INVALID_ARG;
    if ((long long)B * Hq > 65535) return HIFA4_ERR_UNSUPPORTED;
    return from_cuda(launch_calibrate(dtype == HIFA4_BF16, q, k, B, Hq, Hkv, N, D, alpha, s, s_inv,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_quantize_qkv_ex(const void* q, const void* k, const void* v, hifa4_dtype dtype, int B, int Hq,
                                   int Hkv, int Nq, int Nkv, int D, const hifa4_prequant* pre,
                                   const hifa4_packed* out, hifa4_stream_t stream) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (dtype != HIFA4_F16 && dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (!shape_ok(B, Hq, Hkv, Nq, Nkv, D)) return HIFA4_ERR_UNSUPPORTED;
    const void* ptrs[9] = {q, k, v, out->qc, out->qs, out->kc, out->ks, out->vtc, out->vts};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned16(p)) return HIFA4_ERR_INVALID_ARG;
    hifa4_prequant x{};
    if (pre != nullptr) x = *pre;
    const hifa4_status pc = check_prequant(x, true, true);
    if (pc != HIFA4_OK) return pc;
    if ((long long)B * Hq * Nq > INT32_MAX || (long long)B * Hkv * Nkv > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    const Sizes sz = sizes_of(B, Hq, Hkv, Nq, Nkv, D);
    QuantArgs a{};
    a.bf16 = dtype == HIFA4_BF16;
    a.D = D;
    a.G = Hq / Hkv;
    a.hkv = Hkv;
    a.nq = Nq;
    a.nkv = Nkv;
    a.nkv_in = Nkv;
    a.kv_start = 0;
    a.tiles_q = sz.Tq;
    a.n_groups = (long long)B * Hkv;
    a.q = q;
    a.k = k;
    a.v = v;
    set_prequant(a, x);
    a.qc = static_cast<uint8_t*>(out->qc);
    a.qs = static_cast<uint8_t*>(out->qs);
    a.kc = static_cast<uint8_t*>(out->kc);
    a.ks = static_cast<uint8_t*>(out->ks);
    a.vtc = static_cast<uint8_t*>(out->vtc);
    a.vts = static_cast<uint8_t*>(out->vts);
    a.wait_limit_ns = wait_limit_ns();
    a.stall_loads = g_stall_loads.load();
    return from_cuda(launch_quantize_qkv(a, reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_quantize_q(const void* q, hifa4_dtype dtype, int B, int Hq, int Hkv, int Nq, int D,
                              const hifa4_prequant* pre, const hifa4_packed* out, hifa4_stream_t stream) {
    if (q == nullptr || out == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (dtype != HIFA4_F16 && dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (!shape_ok(B, Hq, Hkv, Nq, 128, D)) return HIFA4_ERR_UNSUPPORTED;
    const void* ptrs[3] = {q, out->qc, out->qs};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned16(p)) return HIFA4_ERR_INVALID_ARG;
    hifa4_prequant x{};
    if (pre != nullptr) x = *pre;
    if (x.s_bias != nullptr) return HIFA4_ERR_INVALID_ARG;
    const float* mean = x.q_mean;
    if (!aligned16(mean)) return HIFA4_ERR_INVALID_ARG;
    x.q_mean = nullptr;
    x.s_inv = x.s;                                  // only s applies to Q (pairing checked on s alone)
    const hifa4_status pc = check_prequant(x, true, false);
    if (pc != HIFA4_OK) return pc;
    x.s_inv = nullptr;
    x.k_pos = nullptr;
    if ((long long)B * Hq * Nq > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    const Sizes sz = sizes_of(B, Hq, Hkv, Nq, 128, D);
    QuantArgs a{};
    a.bf16 = dtype == HIFA4_BF16;
    a.D = D;
    a.G = Hq / Hkv;
    a.hkv = Hkv;
    a.nq = Nq;
    a.nkv = 0;
    a.nkv_in = 0;                                   // no K / V work
    a.kv_start = 0;
    a.tiles_q = sz.Tq;
    a.n_groups = (long long)B * Hkv;
    a.q = q;
    set_prequant(a, x);
    a.q_mean = mean;
    a.qc = static_cast<uint8_t*>(out->qc);
    a.qs = static_cast<uint8_t*>(out->qs);
    a.wait_limit_ns = wait_limit_ns();
    a.stall_loads = g_stall_loads.load();
    return from_cuda(launch_quantize_qkv(a, reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_quantize_qkv(const void* q, const void* k, const void* v, hifa4_dtype dtype, int B, int Hq, int Hkv,
                                int Nq, int Nkv, int D, const float* s, const float* s_inv, const hifa4_packed* out,
                                hifa4_stream_t stream) {
    hifa4_prequant x{};
    x.s = s;
    x.s_inv = s_inv;
    return hifa4_quantize_qkv_ex(q, k, v, dtype, B, Hq, Hkv, Nq, Nkv, D, &x, out, stream);
}

hifa4_status hifa4_append_kv(const void* k, const void* v, hifa4_dtype dtype, int B, int Hkv, int n_new, int D,
                             const hifa4_prequant* pre, const hifa4_packed* cache, int cache_tokens, int start,
                             hifa4_stream_t stream) {
    if (k == nullptr || v == nullptr || cache == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (dtype != HIFA4_F16 && dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (!shape_ok(B, Hkv, Hkv, 16, cache_tokens, D)) return HIFA4_ERR_UNSUPPORTED;
    if (n_new <= 0 || n_new % 16 != 0 || start < 0 || start % 16 != 0 || (long long)start + n_new > cache_tokens)
        return HIFA4_ERR_INVALID_ARG;
    const void* ptrs[6] = {k, v, cache->kc, cache->ks, cache->vtc, cache->vts};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned16(p)) return HIFA4_ERR_INVALID_ARG;
    hifa4_prequant x{};
    if (pre != nullptr) x = *pre;
    if (x.q_mean != nullptr || x.s_bias != nullptr) return HIFA4_ERR_INVALID_ARG;
    x.s = x.s_inv;                                  // only s_inv applies to K (pairing checked on s_inv alone)
    const hifa4_status pc = check_prequant(x, false, true);
    if (pc != HIFA4_OK) return pc;
    x.s = nullptr;
    if ((long long)B * Hkv * cache_tokens > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    QuantArgs a{};
    a.bf16 = dtype == HIFA4_BF16;
    a.D = D;
    a.G = 1;
    a.hkv = Hkv;
    a.nq = 0;
    a.nkv = cache_tokens;
    a.nkv_in = n_new;
    a.kv_start = start;
    a.tiles_q = 0;
    a.n_groups = (long long)B * Hkv;
    a.k = k;
    a.v = v;
    set_prequant(a, x);
    a.kc = static_cast<uint8_t*>(cache->kc);
    a.ks = static_cast<uint8_t*>(cache->ks);
    a.vtc = static_cast<uint8_t*>(cache->vtc);
    a.vts = static_cast<uint8_t*>(cache->vts);
    a.wait_limit_ns = wait_limit_ns();
    a.stall_loads = g_stall_loads.load();
    return from_cuda(launch_quantize_qkv(a, reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_quantize_kv(const void* k, const void* v, hifa4_dtype dtype, int B, int Hkv, int Nkv, int D,
                               const float* s_inv, const hifa4_packed* out, hifa4_stream_t stream) {
    if (out == nullptr) return HIFA4_ERR_INVALID_ARG;
    hifa4_prequant x{};
    x.s_inv = s_inv;
    return hifa4_append_kv(k, v, dtype, B, Hkv, Nkv, D, &x, out, Nkv, 0, stream);
}

hifa4_status hifa4_q_mean(const void* q, hifa4_dtype dtype, int B, int Hq, int Hkv, int Nq, int D,
                          const hifa4_prequant* pre, float* q_mean, hifa4_stream_t stream) {
    if (q == nullptr || q_mean == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (dtype != HIFA4_F16 && dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Hq % Hkv != 0) return HIFA4_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return HIFA4_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(q_mean)) return HIFA4_ERR_INVALID_ARG;
    hifa4_prequant x{};
    if (pre != nullptr) x = *pre;
    x.s_inv = x.s;                                  // only s applies to Q (pairing checked on s alone)
    x.q_mean = nullptr;
    x.s_bias = nullptr;
    const hifa4_status pc = check_prequant(x, true, false);
    if (pc != HIFA4_OK) return pc;
    if ((long long)B * Hq > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    QMeanArgs a{};
    a.bf16 = dtype == HIFA4_BF16;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Nq = Nq;
    a.D = D;
    a.q = q;
    a.s = x.s;
    a.rope_cos = x.rope_cos;
    a.rope_sin = x.rope_sin;
    a.q_pos = x.q_pos;
    a.n_pos = x.n_pos;
    a.mean = q_mean;
    return from_cuda(launch_q_mean(a, reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_attention_fwd(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                 float sm_scale, unsigned flags, hifa4_norm_mode norm, void* o, hifa4_dtype o_dtype,
                                 float* lse, void* workspace, hifa4_stream_t stream) {
    return attention_impl(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse, nullptr, workspace,
                          stream);
}

hifa4_status hifa4_attention_fwd_ex(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                    float sm_scale, unsigned flags, hifa4_norm_mode norm, void* o,
                                    hifa4_dtype o_dtype, float* lse, const hifa4_attention_extras* extras,
                                    void* workspace, hifa4_stream_t stream) {
    return attention_impl(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse, extras, workspace,
                          stream);
}

hifa4_status hifa4_attention_fwd_debug(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                       float sm_scale, unsigned flags, hifa4_norm_mode norm, void* o,
                                       hifa4_dtype o_dtype, float* lse, uint8_t* p_codes, uint8_t* p_scales,
                                       void* workspace, hifa4_stream_t stream) {
    if (p_codes == nullptr || p_scales == nullptr) return HIFA4_ERR_INVALID_ARG;
    hifa4_attention_extras x{};
    x.p_codes = p_codes;
    x.p_scales = p_scales;
    return attention_impl(in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse, &x, workspace, stream);
}

hifa4_status hifa4_attention_fwd_q(const void* q, hifa4_dtype q_dtype, const float* s, const hifa4_packed* kv, int B,
                                   int Hq, int Hkv, int Nq, int Nkv, int D, float sm_scale, unsigned flags,
                                   hifa4_norm_mode norm, void* o, hifa4_dtype o_dtype, float* lse, void* workspace,
                                   hifa4_stream_t stream) {
    if (q == nullptr || kv == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (q_dtype != HIFA4_F16 && q_dtype != HIFA4_BF16) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(s)) return HIFA4_ERR_INVALID_ARG;
    // the Q entries of the packed struct are not read: stand-ins keep the shared checks
    hifa4_packed in = *kv;
    in.qc = in.kc;
    in.qs = in.ks;
    const hifa4_status chk = check_attention_args(&in, B, Hq, Hkv, Nq, Nkv, D, sm_scale, flags, norm, o, o_dtype, lse);
    if (chk != HIFA4_OK) return chk;
    if (D != 128 || decode_mode(Hq, Hkv, Nq, Nkv, D, flags)) return HIFA4_ERR_UNSUPPORTED;
    if (workspace == nullptr || !aligned16(workspace)) return HIFA4_ERR_INVALID_ARG;
    const bool causal = (flags & HIFA4_CAUSAL) != 0;
    const long long rows_k = (long long)B * Hkv * Nkv, rows_v = (long long)B * Hkv * D;
    const Sizes sz = sizes_of(B, Hq, Hkv, Nq, Nkv, D);
    const int nqt = 2;
    const long long n_work = (long long)B * Hkv * ((sz.Tq + nqt - 1) / nqt);
    // Q as rows of D 16-bit elements (256 bytes), loaded as two 128-byte column
    // halves per 128-row tile with the 128-byte swizzle
    const long long rows_q = (long long)B * Hq * Nq;
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, q, (uint64_t)D * 2, (uint64_t)rows_q, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tk, kv->kc, (uint64_t)D / 2, (uint64_t)rows_k, D / 2, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&tv, kv->vtc, 64, (uint64_t)rows_v * (Nkv / 128), 64, D, CU_TENSOR_MAP_SWIZZLE_64B))
        return from_cuda(cudaErrorInvalidValue);
    AttnParams p{};
    p.ks = static_cast<const uint8_t*>(kv->ks);
    p.vts = static_cast<const uint8_t*>(kv->vts);
    p.o = o;
    p.lse = lse;
    p.q_scale = s;
    p.q_bf16 = q_dtype == HIFA4_BF16 ? 1 : 0;
    p.status = static_cast<uint32_t*>(workspace);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.G = Hq / Hkv;
    p.Tq = sz.Tq;
    p.n_kv_tiles = Nkv / 128;
    p.n_work = (int)n_work;
    p.heavy_first = (causal && Nq % (128 * nqt) == 0) ? 1 : 0;
    p.c = (float)((double)sm_scale * 1.4426950408889634074);
    p.wait_limit_ns = wait_limit_ns();
    p.stall_loads = g_stall_loads.load();
    const int out = o_dtype == HIFA4_F16 ? 0 : (o_dtype == HIFA4_BF16 ? 1 : 2);
    return from_cuda(launch_attention(&tq, &tk, &tv, p, D, (int)norm, causal, out, 3, false,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_tile_stats(const float* tile_sums, int B, int Hq, int Nq, int Nkv, float* eps_bar,
                              hifa4_stream_t stream) {
    if (tile_sums == nullptr || eps_bar == nullptr) return HIFA4_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Nq <= 0 || Nkv <= 0 || Nkv % 128 != 0) return HIFA4_ERR_INVALID_ARG;
    if (!aligned16(tile_sums) || (reinterpret_cast<uintptr_t>(eps_bar) & 3u)) return HIFA4_ERR_INVALID_ARG;
    if ((long long)B * Hq > INT32_MAX) return HIFA4_ERR_UNSUPPORTED;
    return from_cuda(launch_tile_stats(reinterpret_cast<const float2*>(tile_sums), B * Hq, Nq, Nkv / 128, eps_bar,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

hifa4_status hifa4_get_status(void* workspace, hifa4_stream_t stream) {
    if (workspace == nullptr) return HIFA4_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (from_cuda(cudaStreamSynchronize(st)) != HIFA4_OK) return HIFA4_ERR_CUDA;
    uint32_t word = 0, qword = 0;
    if (from_cuda(cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost)) != HIFA4_OK)
        return HIFA4_ERR_CUDA;
    if (word != 0 && from_cuda(cudaMemset(workspace, 0, sizeof(word))) != HIFA4_OK) return HIFA4_ERR_CUDA;
    if (from_cuda(take_quantize_status(&qword)) != HIFA4_OK) return HIFA4_ERR_CUDA;
    if (word == 0) word = qword;
    return word == 0 ? HIFA4_OK : (hifa4_status)word;
}

long long hifa4_debug_set_wait_limit(long long limit_ns, int stall_loads) {
    g_stall_loads.store(stall_loads ? 1 : 0);
    const long long prev = g_wait_limit_ns.exchange(limit_ns > 0 ? limit_ns : 0);
    return prev > 0 ? prev : (long long)kDefaultWaitNs;
}

const char* hifa4_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

const char* hifa4_status_string(hifa4_status s) {
    switch (s) {
        case HIFA4_OK: return "ok";
        case HIFA4_ERR_INVALID_ARG: return "invalid argument";
        case HIFA4_ERR_UNSUPPORTED: return "unsupported shape or option";
        case HIFA4_ERR_CUDA: return "CUDA error";
        case HIFA4_ERR_TIMEOUT: return "bounded wait expired inside a kernel";
        default: return "unknown status";
    }
}

int hifa4_version(void) { return 100; }

}  // extern "C"
