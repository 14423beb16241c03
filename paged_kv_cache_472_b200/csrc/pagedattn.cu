// C ABI of libpagedattn: argument validation, the host-side planner and
// kernel dispatch.  Declarations and contracts live in include/pagedattn.h.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "append.cuh"
#include "decode.cuh"
#include "prefill.cuh"

namespace {

thread_local char g_msg[256] = "";

pa_status fail(pa_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

pa_status ok() {
    g_msg[0] = '\0';
    return PA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int elem_bytes(int dtype) { return dtype == PA_DTYPE_F32 ? 4 : 2; }
bool tensor_core_dtype(int dtype) { return dtype == PA_DTYPE_BF16 || dtype == PA_DTYPE_F16; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kSmemLimit = 232448;     // opt-in shared memory per CTA on sm_100 (static + dynamic)
// the decode kernel's static shared memory: control block, lengths and prefix-sum caches
constexpr int kPrefillStaticSmem = 3072;  // barriers, row exchange, tensor-memory address, abort flag
constexpr int kStaticSmem = (int)sizeof(pa::DecodeCtl) + 4 * pa::kLensCache + 8 * (pa::kPrefixCache + 1) + 256;
constexpr size_t kWsHeader = 256;      // error word, dynamic-list counters
constexpr size_t kWsGrab = 64;         // header offset of the grains-handed-out counter
constexpr size_t kWsGrabDone = 128;    // header offset of the finished-CTA counter
// Balanced mode: share of each vr's tiles handed out at run time (0 = none).
// Grains of ~1/8 of a CTA's share cost a cold block-table fetch and a partial
// each; measured on the Qwen3-0.6B-shaped batch they lose more than the
// balance gains, so the planner leaves the list static unless asked.
constexpr int kDynamicShare = 0;
constexpr int kMaxDynamicShare = 64;
constexpr int kStageTargetBytes = 32768;  // K bytes per stage (V the same)

// Merge counters of the workspace: one int per (request, head group).
size_t counters_bytes(int B, int NHG) { return round_up((size_t)B * NHG * 4, 256); }
// Merge-grid records (plans with split_merge): one per (request, head group).
size_t records_bytes(int B, int NHG) { return round_up((size_t)B * NHG * sizeof(pa::MergeRecord), 256); }
constexpr int kMaxStages = 4;

pa_status check_shape(const pa_shape *s) {
    if (!s) return fail(PA_ERR_INVALID_ARG, "shape is NULL");
    if (s->B < 0) return fail(PA_ERR_INVALID_ARG, "B=%d < 0", s->B);
    if (s->Hq <= 0 || s->Hkv <= 0) return fail(PA_ERR_INVALID_ARG, "Hq=%d Hkv=%d must be > 0", s->Hq, s->Hkv);
    if (s->Hq % s->Hkv) return fail(PA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", s->Hq, s->Hkv);
    if (s->D <= 0 || s->block_size <= 0 || s->num_blocks <= 0 || s->max_blocks_per_seq <= 0)
        return fail(PA_ERR_INVALID_ARG, "D, block_size, num_blocks, max_blocks_per_seq must be > 0");
    if (s->dtype != PA_DTYPE_F32 && s->dtype != PA_DTYPE_BF16 && s->dtype != PA_DTYPE_F16)
        return fail(PA_ERR_INVALID_ARG, "dtype=%d is not a pa_dtype", s->dtype);
    if ((int64_t)s->num_blocks * s->block_size > INT32_MAX)
        return fail(PA_ERR_UNSUPPORTED, "num_blocks*block_size exceeds the int32 slot range");
    if ((int64_t)s->max_blocks_per_seq * s->block_size > INT32_MAX)
        return fail(PA_ERR_UNSUPPORTED, "max_blocks_per_seq*block_size exceeds int32");
    return PA_OK;
}

// ---------------------------------------------------------------------------
// decode kernel variants.  bf16: tensor-core engine (D, units per warp);
// fp32: CUDA-core engine (D, heads per unit, units per warp).
using KernelFn = void (*)(const pa::DecodeParams);

template <int D>
KernelFn pick_core(int hc, int upw) {
#define PA_CASE(H, U) \
    if (hc == H && upw == U) return pa::paged_decode_kernel<float, D, pa::CoreEngine<float, D, H, U>>;
    PA_CASE(1, 1) PA_CASE(2, 1) PA_CASE(4, 1) PA_CASE(1, 2) PA_CASE(2, 2) PA_CASE(4, 2) PA_CASE(1, 4) PA_CASE(2, 4)
#undef PA_CASE
    return nullptr;
}

template <typename T, int D>
KernelFn pick_mma(int upw, int ts) {
    if (upw == 1 && ts > 1) return pa::paged_decode_kernel<T, D, pa::MmaEngine<T, D, 1, true>>;
    if (upw == 1) return pa::paged_decode_kernel<T, D, pa::MmaEngine<T, D, 1>>;
    if (upw == 2) return pa::paged_decode_kernel<T, D, pa::MmaEngine<T, D, 2>>;
    return nullptr;
}

// tcgen05 engine: one KV head per work item and all its G query heads in one
// tensor-core tile (heads_per_unit = G >= 16 names it in the plan)
template <typename T>
KernelFn pick_tc(int G) {
    if (G == 16) return pa::paged_decode_kernel<T, 128, pa::TcEngine<T, 16>>;
    if (G == 32) return pa::paged_decode_kernel<T, 128, pa::TcEngine<T, 32>>;
    if (G == 64) return pa::paged_decode_kernel<T, 128, pa::TcEngine<T, 64>>;
    return nullptr;
}

KernelFn pick_kernel(int dtype, int D, int hc, int upw, int ts) {
    if (hc >= 16) {
        if (D != 128 || upw != 1 || ts != 1) return nullptr;
        if (dtype == PA_DTYPE_BF16) return pick_tc<__nv_bfloat16>(hc);
        if (dtype == PA_DTYPE_F16) return pick_tc<__half>(hc);
        return nullptr;
    }
    if (dtype == PA_DTYPE_BF16)
        return D == 64 ? pick_mma<__nv_bfloat16, 64>(upw, ts)
                       : (D == 128 ? pick_mma<__nv_bfloat16, 128>(upw, ts) : nullptr);
    if (dtype == PA_DTYPE_F16)
        return D == 64 ? pick_mma<__half, 64>(upw, ts) : (D == 128 ? pick_mma<__half, 128>(upw, ts) : nullptr);
    return D == 64 ? pick_core<64>(hc, upw) : (D == 128 ? pick_core<128>(hc, upw) : nullptr);
}

KernelFn pick_merge(int dtype, int D) {
    if (dtype == PA_DTYPE_BF16)
        return D == 64 ? pa::paged_merge_kernel<__nv_bfloat16, 64> : pa::paged_merge_kernel<__nv_bfloat16, 128>;
    if (dtype == PA_DTYPE_F16) return D == 64 ? pa::paged_merge_kernel<__half, 64> : pa::paged_merge_kernel<__half, 128>;
    return D == 64 ? pa::paged_merge_kernel<float, 64> : pa::paged_merge_kernel<float, 128>;
}

std::mutex g_attr_mu;

pa_status ensure_smem_attr(KernelFn fn, int bytes) {
    // cudaFuncSetAttribute is cheap but not free; remember the largest size set per kernel.
    static struct {
        KernelFn fn;
        int bytes;
    } seen[64];
    static int nseen = 0;
    std::lock_guard<std::mutex> lk(g_attr_mu);
    for (int i = 0; i < nseen; ++i)
        if (seen[i].fn == fn && seen[i].bytes >= bytes) return PA_OK;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    for (int i = 0; i < nseen; ++i)
        if (seen[i].fn == fn) {
            seen[i].bytes = bytes;
            return PA_OK;
        }
    if (nseen < 64) seen[nseen++] = {fn, bytes};
    return PA_OK;
}

struct Layout {
    uint32_t off_bar, off_q, off_stage, off_scratch, off_comb, total;
    uint32_t comb_stride;
};

// shared-memory layout of one decode CTA
Layout smem_layout(int dtype, int D, int stages, uint32_t q_bytes, uint32_t half_bytes, int hc, int tsplit,
                   int nhvr) {
    Layout l;
    if (hc >= 16) {
        // tcgen05 engine: q slots and stages 1024-aligned (128-byte swizzled
        // boxes), then the softmax warps' exchange area: red[2][4][G],
        // running maxima [4][G] and rescale factors [4][G]
        l.off_bar = 0;
        const uint32_t bar_bytes = (uint32_t)round_up((2 * stages + 4 + pa::kMaxPending + 2 + pa::kMergeRing + pa::kTcBars) * 8, 128);
        l.off_q = (uint32_t)round_up(bar_bytes, 1024);
        l.off_stage = (uint32_t)round_up(l.off_q + 2 * q_bytes, 1024);
        l.off_scratch = l.off_stage + (uint32_t)stages * 2 * half_bytes;
        l.off_comb = (uint32_t)round_up(l.off_scratch + 16u * hc * 4u, 128);
        l.comb_stride = 0;
        l.total = l.off_comb + 1024;
        return l;
    }
    const bool mma = tensor_core_dtype(dtype);
    l.off_bar = 0;
    // full/empty per stage, q full/empty, piece-done per pending piece, arrivals done,
    // consumer barrier, the final merge's copy ring
    const uint32_t bar_bytes = (uint32_t)round_up((2 * stages + 4 + pa::kMaxPending + 2 + pa::kMergeRing) * 8, 128);
    l.off_q = bar_bytes;
    l.off_stage = (uint32_t)round_up(l.off_q + 2 * q_bytes, 1024);
    l.off_scratch = (uint32_t)round_up(l.off_stage + (size_t)stages * 2 * half_bytes, 128);
    const uint32_t scratch = mma ? 0u : (uint32_t)(pa::kConsumerWarps * 2 * pa::kSubTile * hc * 4);
    l.off_comb = (uint32_t)round_up(l.off_scratch + scratch, 128);
    const uint32_t comb_floats = mma ? (uint32_t)(4 * (D / 16) * 32 + 4 * 32) : (uint32_t)(hc * D + 8);
    l.comb_stride = comb_floats * 4;
    const uint32_t comb = tsplit > 1 ? pa::kConsumerWarps * l.comb_stride : 0;
    // + 1024: the kernel rounds its dynamic base up to a 1024-byte boundary
    l.total = (uint32_t)round_up(l.off_comb + comb, 128) + 1024;
    return l;
}

// ---------------------------------------------------------------------------
pa_status launch_append(const void *k_new, const void *v_new, const int32_t *slot_mapping, void *k_cache,
                        void *v_cache, const pa_shape *s, int32_t *device_error, cudaStream_t stream) {
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)
        return fail(PA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "value tensors must be 16-byte aligned");
    const int64_t token_bytes = (int64_t)s->Hkv * s->D * elem_bytes(s->dtype);
    if (token_bytes % 16)
        return fail(PA_ERR_UNSUPPORTED, "Hkv*D*elem=%lld is not a multiple of 16", (long long)token_bytes);
    const int vec = (int)(token_bytes / 16);
    const int64_t total = (int64_t)s->B * vec;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    pa::kv_append_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        (const uint4 *)k_new, (const uint4 *)v_new, slot_mapping, (uint4 *)k_cache, (uint4 *)v_cache, s->B, vec,
        (int64_t)s->num_blocks * s->block_size, device_error);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "append launch: %s", cudaGetErrorString(e));
    return PA_OK;
}

struct Mapping {
    int HG, HC, UPW, TS;
};

// Head group HG (KV heads per work item), heads per warp unit HC, units per
// warp UPW and warps per unit TS (token split) for one shape and engine.
// The tcgen05 engine takes bf16 / fp16 shapes with D = 128 and a group of
// 16, 32 or 64 query heads per KV head, with tiles of 128 tokens (so fixed
// partitions must be multiples of 128).
bool tc_engine_shape(const pa_shape *s, int partition_tokens) {
    const int G = s->Hq / s->Hkv;
    return tensor_core_dtype(s->dtype) && s->D == 128 && (G == 16 || G == 32 || G == 64) &&
           partition_tokens % pa::kTcTile == 0;
}

bool choose_mapping(const pa_shape *s, Mapping &m) {
    const int G = s->Hq / s->Hkv;
    const int e = elem_bytes(s->dtype);
    const bool mma = tensor_core_dtype(s->dtype);
    for (int hg = s->Hkv; hg >= 1; --hg) {
        if (s->Hkv % hg || hg * s->D * e > 2048) continue;
        if (mma) {
            // a unit is one KV head and up to 8 of its query heads (one n=8 tile)
            const int hc = G < 8 ? G : 8;
            const int U = hg * (G / hc);
            if (U >= 8 && U % 8 == 0 && U / 8 <= 2) {
                m = {hg, hc, U / 8, 1};
                return true;
            }
            if (U < 8 && 8 % U == 0) {
                m = {hg, hc, 1, 8 / U};
                return true;
            }
            continue;
        }
        for (int hc = 4; hc >= 1; hc >>= 1) {
            if (G % hc) continue;
            const int U = hg * (G / hc);
            if (U >= 8) {
                if (U % 8) continue;
                const int upw = U / 8;
                if (upw > 4 || upw * hc > 8 || (upw == 4 && hc > 2)) continue;
                m = {hg, hc, upw, 1};
                return true;
            }
        }
        const int U = hg * G;  // HC = 1
        if (U < 8 && 8 % U == 0) {
            m = {hg, 1, 1, 8 / U};
            return true;
        }
    }
    return false;
}

uint32_t row_pitch_of(const pa_shape *, uint32_t row_bytes) { return row_bytes; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
PFN_cuTensorMapEncodeTiled encode_fn() {
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(f);
    });
    return fn;
}

// [d, token row, head] view of a bf16 pool [num_blocks, bs, Hkv, D]; the box
// {64, br, HG} lands head-major ([head][row][64]) with the 128-byte swizzle.
pa_status encode_pool_map(CUtensorMap *map, const void *pool, const pa_shape *s, int br, int hg) {
    PFN_cuTensorMapEncodeTiled enc = encode_fn();
    if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[3] = {(cuuint64_t)s->D, (cuuint64_t)s->num_blocks * (cuuint64_t)s->block_size, (cuuint64_t)s->Hkv};
    cuuint64_t strides[2] = {(cuuint64_t)s->Hkv * s->D * 2, (cuuint64_t)s->D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)br, (cuuint32_t)hg};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt =
        s->dtype == PA_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = enc(map, dt, 3, const_cast<void *>(pool), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PA_OK;
}

// [d, request*head] view of q [B, Hq, D]; the box {64, nh} lands as
// [head][128 B] with the 128-byte swizzle (one box per 64-wide d-chunk).
pa_status encode_q_map(CUtensorMap *map, const void *q, const pa_shape *s, int nh) {
    PFN_cuTensorMapEncodeTiled enc = encode_fn();
    if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {(cuuint64_t)s->D, (cuuint64_t)s->B * (cuuint64_t)s->Hq};
    cuuint64_t strides[1] = {(cuuint64_t)s->D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)nh};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        s->dtype == PA_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = enc(map, dt, 2, const_cast<void *>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)r);
    return PA_OK;
}

int log2i(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return l;
}

// The planner proper (pa_plan without the status-message reset).
pa_status plan_internal(const pa_shape *s, int32_t max_context_len, int32_t partition_tokens, int32_t num_sms,
                        pa_plan_t *plan) {
    if (!plan) return fail(PA_ERR_INVALID_ARG, "plan_out is NULL");
    if (pa_status st = check_shape(s)) return st;
    const int cap = s->max_blocks_per_seq * s->block_size;
    if (max_context_len < 0 || max_context_len > cap)
        return fail(PA_ERR_INVALID_ARG, "max_context_len=%d outside [0, %d]", max_context_len, cap);
    if (partition_tokens < 0) return fail(PA_ERR_INVALID_ARG, "partition_tokens=%d < 0", partition_tokens);
    if (s->D != 64 && s->D != 128) return fail(PA_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", s->D);
    if (!pow2(s->block_size) || s->block_size < 16 || s->block_size > 256)
        return fail(PA_ERR_UNSUPPORTED, "block_size=%d (supported: powers of two in [16, 256])", s->block_size);
    const int G = s->Hq / s->Hkv;
    if (!pow2(G) || G > 64) return fail(PA_ERR_UNSUPPORTED, "GQA group %d (supported: powers of two <= 64)", G);
    const int e = elem_bytes(s->dtype);

    if (num_sms <= 0) {
        int dev = 0;
        cudaError_t ce = cudaGetDevice(&dev);
        if (ce == cudaSuccess) ce = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (ce != cudaSuccess) return fail(PA_ERR_CUDA, "querying the SM count: %s", cudaGetErrorString(ce));
    }

    Mapping mp;
    const bool tc = tc_engine_shape(s, partition_tokens);
    if (tc) {
        mp = {1, G, 1, 1};
    } else if (!choose_mapping(s, mp)) {
        return fail(PA_ERR_UNSUPPORTED, "no warp mapping for Hq=%d Hkv=%d D=%d", s->Hq, s->Hkv, s->D);
    }
    const int HG = mp.HG, HC = mp.HC, UPW = mp.UPW, TS = mp.TS;
    const int NHvr = HG * G;
    const int NHG = s->Hkv / HG;
    const uint32_t row_bytes = (uint32_t)(HG * s->D * e);
    const uint32_t pitch = row_pitch_of(s, row_bytes);
    const uint32_t q_bytes = (uint32_t)(NHvr * s->D * e);

    int ST = 16;
    while (ST * 2 <= 256 && (uint32_t)(ST * 2) * row_bytes <= (uint32_t)kStageTargetBytes) ST *= 2;
    if (tc) ST = pa::kTcTile;  // M of the S product
    int mode = PA_SPLIT_BALANCED;
    if (partition_tokens > 0) {
        if (partition_tokens % 16)
            return fail(PA_ERR_INVALID_ARG, "partition_tokens=%d is not a multiple of 16", partition_tokens);
        mode = PA_SPLIT_FIXED;
        while (partition_tokens % ST) ST /= 2;  // tiles must not straddle partitions
    }
    int stages = 0;
    Layout lay{};
    for (;;) {
        const uint32_t half = (uint32_t)ST * pitch;
        for (stages = kMaxStages; stages >= 2; --stages) {
            lay = smem_layout(s->dtype, s->D, stages, q_bytes, half, HC, TS, NHvr);
            if (lay.total + kStaticSmem <= (uint32_t)kSmemLimit) break;
        }
        if (stages >= 2) break;
        if (ST == 16 || tc) return fail(PA_ERR_UNSUPPORTED, "shared memory too small for this shape");
        ST /= 2;
    }

    memset(plan, 0, sizeof *plan);
    plan->mode = mode;
    plan->partition_tokens = mode == PA_SPLIT_FIXED ? partition_tokens : 0;
    plan->num_ctas = num_sms;
    plan->tile_tokens = ST;
    plan->stages = stages;
    plan->head_group = HG;
    plan->heads_per_unit = HC;
    plan->units_per_warp = UPW;
    plan->warps_per_unit = TS;
    plan->max_context_len = max_context_len;
    plan->smem_bytes = (int32_t)lay.total;
    plan->shape = *s;
    if (mode == PA_SPLIT_BALANCED) {
        // static piece (vr v, slice r): slot v + r; dynamic piece (vr v, grain j):
        // NV + C + v + j with j < J <= 8*C*share/256 + 1
        const int64_t NV = (int64_t)s->B * NHG, C = num_sms;
        const bool dyn = s->B <= pa::kPrefixCache && s->B <= pa::kLensCache;
        plan->dynamic_share = dyn ? kDynamicShare : 0;
        // slots for the largest share a caller may set in the plan
        const int64_t Jmax = 8 * C * kMaxDynamicShare / 256 + 1;
        plan->max_slots = dyn ? 2 * NV + C + Jmax : NV + C;
    } else {
        // one partial per (vr, slice) it touches, as in the static list above
        plan->max_slots = (int64_t)s->B * NHG + num_sms;
    }
    // a second grid merges the split requests when each is likely spread over many CTAs
    plan->split_merge = (s->B > 0 && (int64_t)num_sms >= 8 * (int64_t)s->B * NHG) ? 1 : 0;
    const size_t slot_floats = (size_t)NHvr * s->D + round_up(2 * NHvr, 4);
    const size_t counters = counters_bytes(s->B, NHG);
    const size_t records = plan->split_merge ? records_bytes(s->B, NHG) : 0;
    plan->workspace_bytes = kWsHeader + counters + records + (size_t)plan->max_slots * slot_floats * 4;
    return PA_OK;
}


// A plan passed to a decode call must be what the planner gives for its own
// recorded inputs (shape, max_context_len, partition size, CTA count); only
// dynamic_share and flags are the caller's to set.  Everything the launch
// derives from the plan (kernel variant, grid, shared-memory layout,
// workspace offsets) is therefore consistent before anything is queued.
pa_status check_plan(const pa_shape *s, const pa_plan_t *plan) {
    if (!plan) return fail(PA_ERR_INVALID_ARG, "plan is NULL");
    if (memcmp(&plan->shape, s, sizeof *s) != 0) return fail(PA_ERR_INVALID_ARG, "plan was made for another shape");
    if (plan->num_ctas <= 0 || (plan->mode != PA_SPLIT_BALANCED && plan->mode != PA_SPLIT_FIXED))
        return fail(PA_ERR_INVALID_ARG, "plan is inconsistent");
    pa_plan_t ref;
    const int pt = plan->mode == PA_SPLIT_FIXED ? plan->partition_tokens : 0;
    if (plan->mode == PA_SPLIT_FIXED && pt <= 0) return fail(PA_ERR_INVALID_ARG, "plan is inconsistent");
    if (plan_internal(s, plan->max_context_len, pt, plan->num_ctas, &ref) != PA_OK) {
        char why[sizeof g_msg];
        memcpy(why, g_msg, sizeof why);
        return fail(PA_ERR_INVALID_ARG, "plan is inconsistent: %s", why);
    }
    if (ref.mode != plan->mode || ref.partition_tokens != plan->partition_tokens || ref.tile_tokens != plan->tile_tokens ||
        ref.stages != plan->stages || ref.head_group != plan->head_group || ref.heads_per_unit != plan->heads_per_unit ||
        ref.units_per_warp != plan->units_per_warp || ref.warps_per_unit != plan->warps_per_unit ||
        ref.smem_bytes != plan->smem_bytes || ref.max_slots != plan->max_slots ||
        ref.split_merge != plan->split_merge || ref.workspace_bytes != plan->workspace_bytes)
        return fail(PA_ERR_INVALID_ARG, "plan is inconsistent with the planner's output for this shape");
    return PA_OK;
}

// A decode launch, validated and ready to queue.
struct DecodeLaunch {
    pa::DecodeParams p;
    KernelFn fn = nullptr;
    KernelFn merge_fn = nullptr;  // split_merge: the merge grid
    int merge_ctas = 0;
    int smem_bytes = 0;
    int num_ctas = 0;
    int threads = pa::kDecodeThreads;
    bool empty = true;  // nothing to launch (B == 0)
};

// Every host-side check of a decode call, and the kernel parameters it
// implies.  Nothing is queued on the GPU here.  The fused step (k_new !=
// NULL) appends each request's new token in the same launch.
pa_status prepare_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                         const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                         const pa_plan_t *plan, void *workspace, size_t workspace_bytes, const void *k_new,
                         const void *v_new, const int32_t *slot_mapping, DecodeLaunch &L) {
    if (pa_status st = check_plan(s, plan)) return st;
    if (plan->dynamic_share < 0 || plan->dynamic_share > kMaxDynamicShare ||
        (plan->dynamic_share > 0 && (plan->mode != PA_SPLIT_BALANCED || s->B > pa::kPrefixCache)))
        return fail(PA_ERR_INVALID_ARG, "dynamic_share=%d outside [0, %d] or not available for this plan",
                    plan->dynamic_share, kMaxDynamicShare);
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
    if (plan->flags & ~(PA_PLAN_NO_SPECULATION | PA_PLAN_TEST_MISGUESS | PA_PLAN_TEST_STALL))
        return fail(PA_ERR_INVALID_ARG, "unknown plan flags %#x", plan->flags);
    if (!workspace) return fail(PA_ERR_WORKSPACE, "workspace is NULL");
    if (workspace_bytes < plan->workspace_bytes)
        return fail(PA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, plan->workspace_bytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    L.empty = s->B == 0;
    if (L.empty) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out)
        return fail(PA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return fail(PA_ERR_INVALID_ARG, "value tensors must be 16-byte aligned");

    const int HC = plan->heads_per_unit, UPW = plan->units_per_warp, TS = plan->warps_per_unit;
    const int G = s->Hq / s->Hkv;
    const int e = elem_bytes(s->dtype);
    KernelFn fn = pick_kernel(s->dtype, s->D, HC, UPW, TS);
    if (!fn) return fail(PA_ERR_INVALID_ARG, "plan names no kernel variant");
    const int HG = plan->head_group;
    const int NHvr = HG * G;
    const uint32_t row_bytes = (uint32_t)(HG * s->D * e);
    const uint32_t pitch = row_pitch_of(s, row_bytes);
    const uint32_t half = (uint32_t)plan->tile_tokens * pitch;
    const uint32_t q_bytes = (uint32_t)(NHvr * s->D * e);
    const Layout lay = smem_layout(s->dtype, s->D, plan->stages, q_bytes, half, HC, TS, NHvr);
    if ((int)lay.total != plan->smem_bytes) return fail(PA_ERR_INVALID_ARG, "plan is inconsistent");

    pa::DecodeParams &p = L.p;
    p = pa::DecodeParams{};
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = out;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    const size_t counters = counters_bytes(s->B, s->Hkv / HG);
    p.error = reinterpret_cast<int32_t *>(ws);
    p.grab = reinterpret_cast<int32_t *>(ws + kWsGrab);
    p.grab_done = reinterpret_cast<int32_t *>(ws + kWsGrabDone);
    p.fused = k_new ? 1 : 0;
    p.k_new = k_new;
    p.v_new = v_new;
    p.slot_mapping = slot_mapping;
    p.dyn_num = plan->mode == PA_SPLIT_BALANCED ? plan->dynamic_share : 0;
    p.counters = reinterpret_cast<int32_t *>(ws + kWsHeader);
    const size_t records = plan->split_merge ? records_bytes(s->B, s->Hkv / HG) : 0;
    p.split_merge = plan->split_merge;
    p.records = reinterpret_cast<pa::MergeRecord *>(ws + kWsHeader + counters);
    p.partials = reinterpret_cast<float *>(ws + kWsHeader + counters + records);
    p.qscale = scale * 1.4426950408889634f;
    p.B = s->B;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.bs = s->block_size;
    p.num_blocks = s->num_blocks;
    p.max_blocks = s->max_blocks_per_seq;
    p.G = G;
    p.HG = HG;
    p.NHG = s->Hkv / HG;
    p.NHvr = NHvr;
    p.ST = plan->tile_tokens;
    p.stages = plan->stages;
    p.mode = plan->mode;
    p.part_tiles = plan->mode == PA_SPLIT_FIXED ? plan->partition_tokens / plan->tile_tokens : 1;
    p.num_ctas = plan->num_ctas;
    p.tsplit = TS;
    p.units = HG * (G / HC);
    p.heads_per_unit = HC;
    p.max_slots = plan->max_slots;
    p.slot_floats = (int64_t)NHvr * s->D + (int64_t)round_up(2 * NHvr, 4);
    p.off_bar = lay.off_bar;
    p.off_q = lay.off_q;
    p.off_stage = lay.off_stage;
    p.off_scratch = lay.off_scratch;
    p.off_comb = lay.off_comb;
    p.row_bytes = row_bytes;
    p.row_pitch = pitch;
    p.half_bytes = half;
    p.q_bytes = q_bytes;
    p.comb_stride = lay.comb_stride;
    p.bs_log2 = log2i(s->block_size);
    p.st_log2 = log2i(plan->tile_tokens);
    p.spec = (plan->flags & PA_PLAN_NO_SPECULATION) ? 0 : ((plan->flags & PA_PLAN_TEST_MISGUESS) ? 2 : 1);
    p.test_stall = (plan->flags & PA_PLAN_TEST_STALL) ? 1 : 0;
    p.lens_cached = s->B <= pa::kLensCache ? 1 : 0;
    if (tensor_core_dtype(s->dtype)) {
        const int br = plan->tile_tokens < s->block_size ? plan->tile_tokens : s->block_size;
        p.use_tmap = 1;
        p.br_log2 = log2i(br);
        if (pa_status st = encode_pool_map(&p.tmap_k, k_cache, s, br, HG)) return st;
        if (pa_status st = encode_pool_map(&p.tmap_v, v_cache, s, br, HG)) return st;
    }
    if (HC >= 16) {
        // tcgen05 engine: stages [d-chunk][token row], q staged by its own tensor map
        p.dchunk_major = 1;
        p.use_qmap = 1;
        if (pa_status st = encode_q_map(&p.tmap_q, q, s, NHvr)) return st;
    }
    if (pa_status st = ensure_smem_attr(fn, plan->smem_bytes)) return st;
    L.fn = fn;
    if (plan->split_merge) {
        L.merge_fn = pick_merge(s->dtype, s->D);
        const int64_t ctas = (int64_t)s->B * s->Hq;  // one per (request, query head)
        if (ctas > INT32_MAX) return fail(PA_ERR_UNSUPPORTED, "B*Hq too large for the merge grid");
        L.merge_ctas = (int)ctas;
        if (!L.merge_fn) return fail(PA_ERR_INVALID_ARG, "plan names no merge kernel");
    }
    L.threads = HC >= 16 ? pa::kTcThreads : pa::kDecodeThreads;
    L.smem_bytes = plan->smem_bytes;
    L.num_ctas = plan->num_ctas;
    return PA_OK;
}

// Queue a prepared decode.  The launch may start while the preceding grid on
// the stream finishes (programmatic dependent launch): the kernel waits for
// that grid before its first read of anything it wrote.
pa_status enqueue_decode(const DecodeLaunch &L, cudaStream_t stream) {
    if (L.empty) return PA_OK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)L.num_ctas);
    cfg.blockDim = dim3((unsigned)L.threads);
    cfg.dynamicSmemBytes = (size_t)L.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t ce = cudaLaunchKernelEx(&cfg, L.fn, L.p);
    if (ce == cudaSuccess) ce = cudaGetLastError();
    if (ce != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(ce));
    if (L.merge_fn) {
        // the merge grid, also a programmatic dependent: its CTAs wait for the
        // decode grid's memory before reading any partial
        cfg.gridDim = dim3((unsigned)L.merge_ctas);
        cfg.blockDim = dim3(pa::kMergeThreads);
        cfg.dynamicSmemBytes = 0;
        ce = cudaLaunchKernelEx(&cfg, L.merge_fn, L.p);
        if (ce == cudaSuccess) ce = cudaGetLastError();
        if (ce != cudaSuccess) return fail(PA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(ce));
    }
    return PA_OK;
}

pa_status launch_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                        const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                        const pa_plan_t *plan, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                        const void *k_new, const void *v_new, const int32_t *slot_mapping) {
    DecodeLaunch L;
    if (pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, s, plan, workspace,
                                      workspace_bytes, k_new, v_new, slot_mapping, L))
        return st;
    return enqueue_decode(L, stream);
}

}  // namespace

extern "C" {

int32_t pa_version(void) { return 200; }

const char *pa_status_str(pa_status st) {
    switch (st) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    }
    return "PA_ERR_UNKNOWN";
}

const char *pa_last_error_message(void) { return g_msg; }

pa_status pa_kv_append(const void *k_new, const void *v_new, const int32_t *slot_mapping, void *k_cache,
                       void *v_cache, const pa_shape *s, int32_t *device_error, void *stream) {
    if (pa_status st = check_shape(s)) return st;
    if (s->B == 0) return ok();
    if (pa_status st = launch_append(k_new, v_new, slot_mapping, k_cache, v_cache, s, device_error,
                                     (cudaStream_t)stream))
        return st;
    return ok();
}

pa_status pa_plan(const pa_shape *s, int32_t max_context_len, int32_t partition_tokens, int32_t num_sms,
                  pa_plan_t *plan) {
    if (pa_status st = plan_internal(s, max_context_len, partition_tokens, num_sms, plan)) return st;
    return ok();
}

size_t pa_decode_workspace_size(const pa_plan_t *plan) { return plan ? plan->workspace_bytes : 0; }

pa_status pa_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
    if (!workspace) return fail(PA_ERR_INVALID_ARG, "workspace is NULL");
    cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return ok();
}

pa_status pa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    const int32_t *context_lens, float scale, void *out, const pa_shape *s, const pa_plan_t *plan,
                    void *workspace, size_t workspace_bytes, void *stream) {
    if (pa_status st = check_shape(s)) return st;
    if (pa_status st = launch_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, s, plan, workspace,
                                     workspace_bytes, (cudaStream_t)stream, nullptr, nullptr, nullptr))
        return st;
    return ok();
}

pa_status pa_kv_append_decode(const void *k_new, const void *v_new, const int32_t *slot_mapping, const void *q,
                              void *k_cache, void *v_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                              const pa_plan_t *plan, void *workspace, size_t workspace_bytes, void *stream) {
    if (pa_status st = check_shape(s)) return st;
    if (s->B == 0) return ok();
    if (!workspace || workspace_bytes < (plan ? plan->workspace_bytes : 0) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(PA_ERR_WORKSPACE, "workspace missing, too small or not 256-byte aligned");
    if (!k_new || !v_new || !slot_mapping) return fail(PA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(k_new) || !aligned16(v_new)) return fail(PA_ERR_INVALID_ARG, "value tensors must be 16-byte aligned");
    if (pa_status st = launch_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, s, plan, workspace,
                                     workspace_bytes, (cudaStream_t)stream, k_new, v_new, slot_mapping))
        return st;
    return ok();
}

// ---------------------------------------------------------------------------
// chunked prefill
pa_status pa_prefill_plan(const pa_shape *s, int32_t max_new_tokens, pa_prefill_plan_t *plan) {
    if (!plan) return fail(PA_ERR_INVALID_ARG, "plan_out is NULL");
    if (pa_status st = check_shape(s)) return st;
    if (max_new_tokens < 0 || max_new_tokens > s->max_blocks_per_seq * s->block_size)
        return fail(PA_ERR_INVALID_ARG, "max_new_tokens=%d outside [0, %d]", max_new_tokens,
                    s->max_blocks_per_seq * s->block_size);
    if (!tensor_core_dtype(s->dtype)) return fail(PA_ERR_UNSUPPORTED, "prefill supports bf16 and fp16");
    if (s->D != 64 && s->D != 128) return fail(PA_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", s->D);
    if (!pow2(s->block_size) || s->block_size < 16 || s->block_size > 256)
        return fail(PA_ERR_UNSUPPORTED, "block_size=%d (supported: powers of two in [16, 256])", s->block_size);
    const int G = s->Hq / s->Hkv;
    if (!pow2(G) || G > pa::kPrefillRows)
        return fail(PA_ERR_UNSUPPORTED, "GQA group %d (supported: powers of two <= %d)", G, pa::kPrefillRows);
    if (s->Hkv > 65535 || s->B > 65535) return fail(PA_ERR_UNSUPPORTED, "Hkv or B above 65535");
    const int QT = pa::kPrefillRows / G;
    const int KT = pa::kPrefillKT;
    const uint32_t q_bytes = (uint32_t)pa::kPrefillQTiles * pa::kPrefillRows * s->D * 2;  // both query tiles
    const uint32_t slot = (uint32_t)KT * s->D * 2;
    int nslots = pa::kPrefillMaxSlots;
    uint32_t total = 0;
    for (; nslots >= 2; nslots -= 2) {
        total = q_bytes + (uint32_t)nslots * slot;  // the kernel checks its base is 1024-aligned
        if (total + kPrefillStaticSmem <= (uint32_t)kSmemLimit) break;
    }
    memset(plan, 0, sizeof *plan);
    plan->q_tile = QT;
    plan->kv_tile = KT;
    plan->stages = nslots / 2;
    plan->max_new_tokens = max_new_tokens;
    plan->num_qtiles = (max_new_tokens + pa::kPrefillQTiles * QT - 1) / (pa::kPrefillQTiles * QT);
    plan->smem_bytes = (int32_t)total;
    plan->shape = *s;
    return ok();
}

pa_status pa_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                     const int32_t *context_lens, const int32_t *query_start, float scale, void *out,
                     const pa_shape *s, const pa_prefill_plan_t *plan, int32_t *device_error, void *stream) {
    if (pa_status st = check_shape(s)) return st;
    if (!plan) return fail(PA_ERR_INVALID_ARG, "plan is NULL");
    if (memcmp(&plan->shape, s, sizeof *s) != 0) return fail(PA_ERR_INVALID_ARG, "plan was made for another shape");
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
    if (s->B == 0 || plan->num_qtiles == 0) return ok();
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !out)
        return fail(PA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return fail(PA_ERR_INVALID_ARG, "value tensors must be 16-byte aligned");
    const int G = s->Hq / s->Hkv;
    if (plan->q_tile * G != pa::kPrefillRows || plan->kv_tile != pa::kPrefillKT || plan->stages < 1 ||
        2 * plan->stages > pa::kPrefillMaxSlots)
        return fail(PA_ERR_INVALID_ARG, "plan is inconsistent");
    pa::PrefillParams p{};
    p.q = q;
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.error = device_error;
    // kept above zero: a masked score enters the kernel as -inf and must give
    // weight 0; with scale 0 every score times 2^-100 still rounds 2^x to 1
    p.qscale = std::fmax(std::fabs(scale) * 1.4426950408889634f, 0x1p-100f);
    p.qflip = scale < 0.f ? 0x80008000u : 0u;
    p.B = s->B;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.G = G;
    p.g_log2 = log2i(G);
    p.bs = s->block_size;
    p.bs_log2 = log2i(s->block_size);
    p.num_blocks = s->num_blocks;
    p.max_blocks = s->max_blocks_per_seq;
    p.QT = plan->q_tile;
    const int br = plan->kv_tile < s->block_size ? plan->kv_tile : s->block_size;
    p.br_log2 = log2i(br);
    p.nslots = 2 * plan->stages;
    p.num_qtiles = plan->num_qtiles;
    p.off_ring = (uint32_t)pa::kPrefillQTiles * pa::kPrefillRows * s->D * 2;
    p.slot_bytes = (uint32_t)pa::kPrefillKT * s->D * 2;
    if (pa_status st = encode_pool_map(&p.tmap_k, k_cache, s, br, 1)) return st;
    if (pa_status st = encode_pool_map(&p.tmap_v, v_cache, s, br, 1)) return st;
    using PrefillFn = void (*)(const pa::PrefillParams);
    PrefillFn fn = nullptr;
    if (s->dtype == PA_DTYPE_BF16) fn = s->D == 64 ? pa::paged_prefill_kernel<__nv_bfloat16, 64>
                                                   : pa::paged_prefill_kernel<__nv_bfloat16, 128>;
    else fn = s->D == 64 ? pa::paged_prefill_kernel<__half, 64> : pa::paged_prefill_kernel<__half, 128>;
    {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, plan->smem_bytes);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    // one CTA per (request, CTA tile, KV head); the kernel ranks the pairs by work
    const long long nctas = (long long)plan->num_qtiles * s->Hkv * s->B;
    if (nctas > 0x7FFFFFFFll) return fail(PA_ERR_INVALID_ARG, "too many prefill tiles for one grid");
    dim3 grid((unsigned)nctas);
    fn<<<grid, pa::kPrefillThreads, (size_t)plan->smem_bytes, (cudaStream_t)stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
    return ok();
}

pa_status pa_get_device_error(void *workspace, int32_t clear, int32_t *err_out, void *stream) {
    if (!workspace || !err_out) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(err_out, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && clear) {
        e = cudaMemsetAsync(workspace, 0, sizeof(int32_t), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode for callers that cannot allocate device memory: the workspace is a
// fixed array compiled into this library instead of caller-provided memory.
static constexpr size_t kNoAllocWorkspaceBytes = 16u << 20;  // 16 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_no_alloc_workspace[kNoAllocWorkspaceBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_no_alloc_mu;
void *g_no_alloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the array on the current device.  The host-side name
// g_no_alloc_workspace is only a stand-in, so the address is looked up once
// per device (with that device current) and remembered.
pa_status no_alloc_workspace(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(PA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lk(g_no_alloc_mu);
    if (!g_no_alloc_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_no_alloc_workspace);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        g_no_alloc_ptr[dev] = ptr;
    }
    *out = g_no_alloc_ptr[dev];
    return PA_OK;
}
}  // namespace

extern "C" pa_status pa_decode_no_alloc(const void *q, const void *k_cache, const void *v_cache,
                                        const int32_t *block_tables, const int32_t *context_lens, float scale,
                                        void *out, const pa_shape *s, const pa_plan_t *plan, void *stream) {
    // every host-side check comes before anything touches the array
    if (pa_status st = check_shape(s)) return st;
    if (pa_status st = check_plan(s, plan)) return st;
    if (plan->workspace_bytes > kNoAllocWorkspaceBytes)
        return fail(PA_ERR_WORKSPACE, "this plan needs %zu workspace bytes; the built-in workspace holds %zu",
                    plan->workspace_bytes, kNoAllocWorkspaceBytes);
    if (s->B == 0) return ok();
    void *ws = nullptr;
    if (pa_status st = no_alloc_workspace(&ws)) return st;
    DecodeLaunch L;
    if (pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, s, plan, ws,
                                      kNoAllocWorkspaceBytes, nullptr, nullptr, nullptr, L))
        return st;
    // The array keeps the previous call's contents.  The run-time counters
    // and the merge counters must start at zero (a call that gave up leaves
    // them as they were); the error word (the first four bytes) is left
    // alone, so it gathers the errors of every call until it is read and
    // cleared with pa_no_alloc_device_error.
    const size_t counters = counters_bytes(s->B, s->Hkv / plan->head_group);
    if (kWsHeader + counters > plan->workspace_bytes) return fail(PA_ERR_INVALID_ARG, "plan is inconsistent");
    cudaError_t e = cudaMemsetAsync(static_cast<unsigned char *>(ws) + kWsGrab, 0, kWsHeader - kWsGrab + counters,
                                    (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    if (pa_status st = enqueue_decode(L, (cudaStream_t)stream)) return st;
    return ok();
}

extern "C" pa_status pa_no_alloc_device_error(int32_t clear, int32_t *err_out, void *stream) {
    if (!err_out) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    void *ws = nullptr;
    if (pa_status st = no_alloc_workspace(&ws)) return st;
    return pa_get_device_error(ws, clear, err_out, stream);
}
