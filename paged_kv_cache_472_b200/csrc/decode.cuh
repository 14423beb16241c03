// Paged decode attention for sm_100a (CUDA-core path).
//
// What it computes (BareLLM README: paged KV cache, block table, one-token
// batched decode over unequal histories; MHA/GQA/MQA): for every request b
// and query head h,
//     out[b][h] = sum_t softmax_t(scale * q[b][h] . K_t) V_t ,  t < L_b,
// where K_t / V_t is row t % bs of physical block block_tables[b][t / bs] for
// KV head h / (Hq/Hkv).  The softmax is evaluated with a running maximum and
// sum (the online softmax of the MinivLLM review and the LLAISYS
// self-attention bullet), in fp32, in the base-2 domain (q is pre-scaled by
// scale * log2 e so that every weight is one exp2).
//
// Work decomposition.  A "virtual request" (vr) is one request restricted to
// a group of HG KV heads (HG = Hkv unless one token of all KV heads is too
// large to stage).  Its tokens are cut into tiles of ST tokens.  The tiles of
// all vrs, laid end to end, are divided among persistent CTAs:
//   * balanced mode: CTA c takes tiles [c*NT/C, (c+1)*NT/C) of the flat list,
//     so every CTA moves the same number of bytes whatever the length mix;
//   * fixed mode: the flat list is of partitions of `part_tiles` tiles (the
//     classic flash-decoding split), divided the same way.
// A vr that lies wholly inside one CTA's range is written straight to `out`.
// Otherwise each covering CTA leaves (m, l, o) for its piece in the
// workspace and bumps the vr's counter; the CTA that arrives last combines
// the pieces by log-sum-exp and restores the counter to zero (no CTA ever
// waits for another).
//
// Inside a CTA: warp 8 is a producer that walks the block table and issues
// one bulk asynchronous copy (cp.async.bulk, completion on an mbarrier) per
// block piece into a ring of `stages` shared-memory stages; a tile of a full
// head group is one contiguous run of [ST, HG, D] elements per block, so the
// copy engine moves whole rows and no thread computes addresses per element.
// Warps 0-7 consume: each owns one (KV head, HC query heads) unit, stages the
// q slice of its heads in registers, and for every 16 tokens
//   QK  : lane (slice, token-group) forms 8-element partial dots with packed
//         fp32x2 FMAs; a reduce-scatter across the D/8 slice lanes finishes
//         the dots and leaves each lane a few whole scores;
//   softmax: lanes of each head reduce the tile maximum and sum by shuffles;
//   PV  : every lane accumulates its 8 output elements of all HC heads.
// Shared-memory reads are 16-byte row slices of consecutive lanes, so every
// phase of a warp's load hits 32 distinct banks.
#pragma once

#include "common.cuh"

namespace pa {

constexpr int kConsumerWarps = 8;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kSubTile = 16;  // tokens per online-softmax update

struct DecodeParams {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    void *out;
    float *partials;      // [slots][slot_floats] fp32: o[NHvr][D], m[NHvr], l[NHvr], padding
    int32_t *counters;    // [B * NHG]
    int32_t *error;       // device error word
    float qscale;         // scale * log2(e)
    int32_t B, Hq, Hkv, bs, num_blocks, max_blocks;
    int32_t G, HG, NHG, NHvr;
    int32_t ST;           // tokens per tile (power of two, >= 16)
    int32_t stages;
    int32_t mode;         // PA_SPLIT_BALANCED / PA_SPLIT_FIXED
    int32_t part_tiles;   // fixed mode: tiles per partition
    int32_t num_ctas;
    int32_t tsplit;       // warps sharing one unit (token split)
    int32_t units;        // units per vr = HG * G / HC
    int64_t max_slots;
    int64_t slot_floats;  // NHvr * D + (2 * NHvr rounded up to a multiple of 4)
    uint32_t off_bar, off_q, off_stage, off_scratch, off_comb;
    uint32_t row_bytes;   // HG * D * elem
    uint32_t half_bytes;  // ST * row_bytes (K part of a stage; V part follows)
    uint32_t q_bytes;     // NHvr * D * elem
};

// ---------------------------------------------------------------------------
// element access
template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    // 8 consecutive elements -> 4 float2 pairs
    static __device__ __forceinline__ void load8(const void *p, float2 (&v)[4]) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        v[0] = bf16x2_to_float2(w.x);
        v[1] = bf16x2_to_float2(w.y);
        v[2] = bf16x2_to_float2(w.z);
        v[3] = bf16x2_to_float2(w.w);
    }
    static __device__ __forceinline__ void store8(void *p, const float2 (&v)[4]) {
        uint4 w;
        __nv_bfloat162 t;
        t = __floats2bfloat162_rn(v[0].x, v[0].y);
        w.x = *reinterpret_cast<uint32_t *>(&t);
        t = __floats2bfloat162_rn(v[1].x, v[1].y);
        w.y = *reinterpret_cast<uint32_t *>(&t);
        t = __floats2bfloat162_rn(v[2].x, v[2].y);
        w.z = *reinterpret_cast<uint32_t *>(&t);
        t = __floats2bfloat162_rn(v[3].x, v[3].y);
        w.w = *reinterpret_cast<uint32_t *>(&t);
        *reinterpret_cast<uint4 *>(p) = w;
    }
    static __device__ __forceinline__ void store_zero8(void *p) {
        *reinterpret_cast<uint4 *>(p) = make_uint4(0, 0, 0, 0);
    }
};

template <>
struct Elem<float> {
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ void load8(const void *p, float2 (&v)[4]) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        v[0] = make_float2(a.x, a.y);
        v[1] = make_float2(a.z, a.w);
        v[2] = make_float2(b.x, b.y);
        v[3] = make_float2(b.z, b.w);
    }
    static __device__ __forceinline__ void store8(void *p, const float2 (&v)[4]) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
        reinterpret_cast<float4 *>(p)[1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
    }
    static __device__ __forceinline__ void store_zero8(void *p) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4 *>(p)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
};

// ---------------------------------------------------------------------------
// work list (identical sequence in every warp of a CTA)
__device__ __forceinline__ int clamped_len(const DecodeParams &p, int b) {
    int L = p.context_lens[b];
    const int cap = p.max_blocks * p.bs;
    return L < 0 ? 0 : (L > cap ? cap : L);
}

// work units of a request: tiles (balanced) or partitions (fixed)
__device__ __forceinline__ int units_of_len(const DecodeParams &p, int L) {
    const int tiles = (L + p.ST - 1) / p.ST;
    return p.mode == PA_SPLIT_BALANCED ? tiles : (tiles + p.part_tiles - 1) / p.part_tiles;
}

__device__ __forceinline__ int64_t range_lo(int64_t c, int64_t NT, int64_t C) { return c * NT / C; }

// CTA whose range contains flat unit x
__device__ __forceinline__ int64_t cta_of(int64_t x, int64_t NT, int64_t C) { return ((x + 1) * C - 1) / NT; }

struct Seg {
    int b, hg, L;
    int t_begin, t_end;  // tiles of the vr
    int nparts;          // pieces this vr is split into (1 = whole vr here)
    int64_t slot;        // partial slot when nparts > 1
    int64_t vr_start;    // flat index of the vr's first unit
    int units;           // units of the vr
};

struct SegIter {
    int64_t cur, hi, lo, NT, C;
    int64_t vr_start;
    int b, hg, L, units;

    __device__ __forceinline__ bool next(const DecodeParams &p, Seg &s) {
        while (cur < hi) {
            if (cur >= vr_start + units) {
                vr_start += units;
                if (++hg == p.NHG) {
                    hg = 0;
                    ++b;
                    L = (b < p.B) ? clamped_len(p, b) : 0;
                    units = (b < p.B) ? units_of_len(p, L) : 0;
                    if (b >= p.B) return false;
                }
                continue;
            }
            const int u0 = (int)(cur - vr_start);
            int u1;
            s.b = b;
            s.hg = hg;
            s.L = L;
            s.vr_start = vr_start;
            s.units = units;
            const int tiles = (L + p.ST - 1) / p.ST;
            if (p.mode == PA_SPLIT_BALANCED) {
                const int64_t end = vr_start + units < hi ? vr_start + units : hi;
                u1 = (int)(end - vr_start);
                s.t_begin = u0;
                s.t_end = u1;
                const int64_t c0 = cta_of(vr_start, NT, C);
                const int64_t c1 = cta_of(vr_start + units - 1, NT, C);
                s.nparts = (int)(c1 - c0 + 1);
                s.slot = 2 * (int64_t)blockIdx.x + (cur == lo ? 0 : 1);
            } else {
                u1 = u0 + 1;
                s.t_begin = u0 * p.part_tiles;
                s.t_end = min(tiles, (u0 + 1) * p.part_tiles);
                s.nparts = units;
                s.slot = vr_start + u0;
            }
            cur = vr_start + u1;
            return true;
        }
        return false;
    }
};

struct __align__(16) DecodeCtl {
    int64_t red[kConsumerWarps + 1];
    int64_t total;
    int64_t found_b, found_excl;
    int abort;
    int merge_flag;
};

// ---------------------------------------------------------------------------
// reduce-scatter of N per-lane values across the RL lanes of a slice group
// (lane bits below log2(RL)).  Afterwards lane `sl` holds value indices
// [sl*N/RL, (sl+1)*N/RL) in v[0..), or, when N < RL, index sl / (RL/N) in v[0].
template <int N, int M>
struct ReduceScatter {
    static __device__ __forceinline__ void run(float *v, int lane) {
        if constexpr (M >= 1) {
            if constexpr (N > 1) {
                constexpr int H = N / 2;
                const bool upper = (lane & M) != 0;
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const float send = upper ? v[i] : v[i + H];
                    const float keep = upper ? v[i + H] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
                }
                ReduceScatter<H, M / 2>::run(v, lane);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
                ReduceScatter<1, M / 2>::run(v, lane);
            }
        }
    }
};

template <int N>
struct ReduceScatter<N, 0> {
    static __device__ __forceinline__ void run(float *, int) {}
};

// ---------------------------------------------------------------------------
template <typename T, int D, int HC, int UPW>
struct Consumer {
    static constexpr int RL = D / 8;          // lanes per token row (8 elements each)
    static constexpr int TG = 32 / RL;        // token rows per warp load
    static constexpr int R = kSubTile / TG;   // rounds per sub-tile
    static constexpr int NV = R * HC;         // partial dots per lane
    static constexpr int NVL = NV >= RL ? NV / RL : 1;
    static constexpr int LPH = (32 / HC) < 16 ? (32 / HC) : 16;  // softmax lanes per head
    static constexpr int TPL = kSubTile / LPH;                   // tokens per softmax lane
    static constexpr int E = Elem<T>::kBytes;

    struct Unit {
        float2 q2[HC][4];
        float2 o2[HC][4];
        float m_own, l_own;  // running max / sum of head (lane / LPH), base-2 domain
    };

    // One 16-token sub-tile of one unit.  kst/vst point at token 0 of the
    // sub-tile in the stage; rows are HG*D elements apart.
    static __device__ __forceinline__ void subtile(Unit &u, const unsigned char *kst, const unsigned char *vst,
                                                   int g_local, int nvalid, uint32_t row_bytes, float *s_sm,
                                                   float *p_sm, int lane) {
        const int sl = lane % RL;
        const int tg = lane / RL;
        const uint32_t col = (uint32_t)(g_local * D + sl * 8) * E;

        // ---- QK: partial dots over this lane's 8 elements ----
        float acc[NV];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int tok = r * TG + tg;
            float2 k2[4];
            if (tok < nvalid) {
                Elem<T>::load8(kst + tok * row_bytes + col, k2);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) k2[i] = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int h = 0; h < HC; ++h) {
                float2 a = fmul2(u.q2[h][0], k2[0]);
                a = ffma2(u.q2[h][1], k2[1], a);
                a = ffma2(u.q2[h][2], k2[2], a);
                a = ffma2(u.q2[h][3], k2[3], a);
                acc[h * R + r] = a.x + a.y;
            }
        }
        ReduceScatter<NV, RL / 2>::run(acc, lane);
        // value j of this lane is (head, round) index i = h*R + r
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int i = (NV >= RL) ? sl * NVL + j : sl / (RL / NV);
            const int h = i / R, r = i % R;
            s_sm[h * kSubTile + r * TG + tg] = acc[j];
        }
        __syncwarp();

        // ---- online softmax per head ----
        const int hs = lane / LPH;  // head served by this lane (HC*LPH <= 32)
        const int li = lane % LPH;
        const bool active = hs < HC;
        float sc[TPL];
        float tmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < TPL; ++k) {
            const int tok = li * TPL + k;
            sc[k] = (active && tok < nvalid) ? s_sm[hs * kSubTile + tok] : -INFINITY;
            tmax = fmaxf(tmax, sc[k]);
        }
#pragma unroll
        for (int m = 1; m < LPH; m <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
        const float m_new = fmaxf(u.m_own, tmax);
        const float alpha = exp2f(u.m_own - m_new);  // m_own = -inf at start -> 0
        float psum = 0.f;
#pragma unroll
        for (int k = 0; k < TPL; ++k) {
            const float pk = exp2f(sc[k] - m_new);  // masked: exp2(-inf) = 0
            psum += pk;
            if (active) p_sm[(li * TPL + k) * HC + hs] = pk;
        }
#pragma unroll
        for (int m = 1; m < LPH; m <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, m);
        u.l_own = u.l_own * alpha + psum;
        u.m_own = m_new;
        __syncwarp();

        // ---- rescale and PV ----
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            const float a = __shfl_sync(0xffffffffu, alpha, h * LPH);
            if (a != 1.f) {
                const float2 a2 = make_float2(a, a);
#pragma unroll
                for (int i = 0; i < 4; ++i) u.o2[h][i] = fmul2(u.o2[h][i], a2);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int tok = r * TG + tg;
            if (tok < nvalid) {
                float2 v2[4];
                Elem<T>::load8(vst + tok * row_bytes + col, v2);
                float pv[HC];
                if constexpr (HC == 4) {
                    const float4 t = *reinterpret_cast<const float4 *>(p_sm + tok * HC);
                    pv[0] = t.x; pv[1] = t.y; pv[2] = t.z; pv[3] = t.w;
                } else if constexpr (HC == 2) {
                    const float2 t = *reinterpret_cast<const float2 *>(p_sm + tok * HC);
                    pv[0] = t.x; pv[1] = t.y;
                } else {
#pragma unroll
                    for (int h = 0; h < HC; ++h) pv[h] = p_sm[tok * HC + h];
                }
#pragma unroll
                for (int h = 0; h < HC; ++h) {
                    const float2 p2 = make_float2(pv[h], pv[h]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) u.o2[h][i] = ffma2(v2[i], p2, u.o2[h][i]);
                }
            }
        }
        __syncwarp();
    }

    // sum the output partials of the TG token-groups (lanes with equal slice)
    static __device__ __forceinline__ void reduce_token_groups(Unit &u) {
#pragma unroll
        for (int m = RL; m < 32; m <<= 1) {
#pragma unroll
            for (int h = 0; h < HC; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    u.o2[h][i].x += __shfl_xor_sync(0xffffffffu, u.o2[h][i].x, m);
                    u.o2[h][i].y += __shfl_xor_sync(0xffffffffu, u.o2[h][i].y, m);
                }
        }
    }
};

// ---------------------------------------------------------------------------
template <typename T, int D, int HC, int UPW>
__global__ void __launch_bounds__(kDecodeThreads, 1) paged_decode_kernel(const DecodeParams p) {
    using C = Consumer<T, D, HC, UPW>;
    constexpr int E = Elem<T>::kBytes;
    constexpr int kCombStride = HC * D + 8;  // floats per warp in the token-split combine area
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ DecodeCtl ctl;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int S = p.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + S;
    uint64_t *qfull = empty + S;
    uint64_t *qempty = qfull + 2;
    volatile int *abort_flag = &ctl.abort;
    unsigned char *qarea = smem + p.off_q;
    unsigned char *stage_base = smem + p.off_stage;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], kConsumerWarps);
        }
        ctl.abort = 0;
        ctl.found_b = -1;
        fence_mbarrier_init();
    }

    // ---- prologue: total units and this CTA's starting point ----
    int64_t local = 0;
    for (int b = tid; b < p.B; b += kDecodeThreads) {
        const int raw = p.context_lens[b];
        if (blockIdx.x == 0 && (raw < 0 || raw > p.max_blocks * p.bs)) set_error(p.error, PA_DEVERR_CONTEXT_LEN);
        local += units_of_len(p, clamped_len(p, b));
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) local += __shfl_xor_sync(0xffffffffu, local, m);
    if (lane == 0) ctl.red[warp] = local;
    __syncthreads();
    if (tid == 0) {
        int64_t t = 0;
        for (int w = 0; w <= kConsumerWarps; ++w) t += ctl.red[w];
        ctl.total = t * p.NHG;
    }
    __syncthreads();
    const int64_t NT = ctl.total;
    // ranges are cut among min(num_ctas, NT) CTAs so none is empty; the rest idle
    const int64_t Cn = NT < p.num_ctas ? (NT > 0 ? NT : 1) : p.num_ctas;
    const int64_t lo = (NT > 0 && blockIdx.x < Cn) ? range_lo(blockIdx.x, NT, Cn) : 0;
    const int64_t hi = (NT > 0 && blockIdx.x < Cn) ? range_lo(blockIdx.x + 1, NT, Cn) : 0;

    if (lo < hi) {
        int64_t running = 0;
        for (int base = 0; base < p.B; base += kDecodeThreads) {
            const int b = base + tid;
            const int64_t u = (b < p.B) ? (int64_t)p.NHG * units_of_len(p, clamped_len(p, b)) : 0;
            int64_t x = u;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, x, m);
                if (lane >= m) x += y;
            }
            __syncthreads();  // ctl.red free to overwrite
            if (lane == 31) ctl.red[warp] = x;
            __syncthreads();
            int64_t before = 0, chunk = 0;
            for (int w = 0; w <= kConsumerWarps; ++w) {
                if (w < warp) before += ctl.red[w];
                chunk += ctl.red[w];
            }
            const int64_t excl = running + before + x - u;
            if (u > 0 && excl <= lo && lo < excl + u) {
                ctl.found_b = b;
                ctl.found_excl = excl;
            }
            running += chunk;
            __syncthreads();
            if (ctl.found_b >= 0) break;
        }
    }
    __syncthreads();

    SegIter it;
    it.cur = lo;
    it.hi = hi;
    it.lo = lo;
    it.NT = NT;
    it.C = Cn;
    if (lo < hi) {
        it.b = (int)ctl.found_b;
        it.L = clamped_len(p, it.b);
        it.units = units_of_len(p, it.L);
        it.hg = (int)((lo - ctl.found_excl) / it.units);
        it.vr_start = ctl.found_excl + (int64_t)it.hg * it.units;
    } else {
        it.b = 0;
        it.hg = 0;
        it.L = 0;
        it.units = 0;
        it.vr_start = 0;
    }

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        const uint64_t policy = policy_evict_first();
        const unsigned char *kc = reinterpret_cast<const unsigned char *>(p.k_cache);
        const unsigned char *vc = reinterpret_cast<const unsigned char *>(p.v_cache);
        const unsigned char *qg = reinterpret_cast<const unsigned char *>(p.q);
        const uint32_t row_bytes = p.row_bytes;
        const size_t tok_stride = (size_t)p.Hkv * D * E;  // bytes between token rows in the pool
        Seg s;
        int64_t fill = 0;
        int segk = 0;
        bool ok = true;
        while (ok && it.next(p, s)) {
            const int qb = segk & 1;
            if (!mbar_wait(&qempty[qb], ((segk >> 1) & 1) ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&qfull[qb], p.q_bytes);
                bulk_g2s(qarea + qb * p.q_bytes, qg + ((size_t)s.b * p.Hq + (size_t)s.hg * p.NHvr) * D * E,
                         p.q_bytes, &qfull[qb]);
            }
            const int32_t *table = p.block_tables + (size_t)s.b * p.max_blocks;
            for (int t = s.t_begin; t < s.t_end; ++t) {
                const int stage = (int)(fill % S);
                if (!mbar_wait(&empty[stage], (uint32_t)((fill / S) & 1) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                unsigned char *kdst = stage_base + (size_t)stage * 2 * p.half_bytes;
                unsigned char *vdst = kdst + p.half_bytes;
                const int tok0 = t * p.ST;
                const int ntok = min(p.ST, s.L - tok0);
                if (p.HG == p.Hkv) {
                    // one copy per block piece: rows of all KV heads are contiguous
                    const int jb0 = tok0 / p.bs;
                    const int np = (tok0 + ntok - 1) / p.bs - jb0 + 1;
                    uint32_t bytes = 0;
                    int phys = -1, r0 = 0, nrows = 0, dtok = 0;
                    if (lane < np) {
                        const int j = jb0 + lane;
                        const int tlo = max(tok0, j * p.bs);
                        const int thi = min(tok0 + ntok, (j + 1) * p.bs);
                        phys = table[j];
                        r0 = tlo - j * p.bs;
                        nrows = thi - tlo;
                        dtok = tlo - tok0;
                        if (phys < 0 || phys >= p.num_blocks) {
                            set_error(p.error, PA_DEVERR_BLOCK_ID);
                            phys = -1;
                        } else {
                            bytes = 2u * (uint32_t)nrows * row_bytes;
                        }
                    }
#pragma unroll
                    for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], bytes);
                    __syncwarp();
                    if (phys >= 0) {
                        const size_t src = ((size_t)phys * p.bs + r0) * tok_stride;
                        const uint32_t n = (uint32_t)nrows * row_bytes;
                        bulk_g2s_hint(kdst + dtok * row_bytes, kc + src, n, &full[stage], policy);
                        bulk_g2s_hint(vdst + dtok * row_bytes, vc + src, n, &full[stage], policy);
                    }
                } else {
                    // head group narrower than the pool row: one copy per token
                    uint32_t bytes = 0;
                    for (int i = lane; i < ntok; i += 32) {
                        const int tt = tok0 + i;
                        const int ph = table[tt / p.bs];
                        if (ph < 0 || ph >= p.num_blocks)
                            set_error(p.error, PA_DEVERR_BLOCK_ID);
                        else
                            bytes += 2u * row_bytes;
                    }
#pragma unroll
                    for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], bytes);
                    __syncwarp();
                    for (int i = lane; i < ntok; i += 32) {
                        const int tt = tok0 + i;
                        const int ph = table[tt / p.bs];
                        if (ph < 0 || ph >= p.num_blocks) continue;
                        const size_t src =
                            ((size_t)ph * p.bs + (tt % p.bs)) * tok_stride + (size_t)s.hg * row_bytes;
                        bulk_g2s_hint(kdst + i * row_bytes, kc + src, row_bytes, &full[stage], policy);
                        bulk_g2s_hint(vdst + i * row_bytes, vc + src, row_bytes, &full[stage], policy);
                    }
                }
                ++fill;
            }
            ++segk;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
        }
        // Let every copy this warp issued land before the CTA can retire.
        volatile int never = 0;
        for (int64_t k = fill - S > 0 ? fill - S : 0; k < fill; ++k)
            mbar_wait(&full[k % S], (uint32_t)((k / S) & 1), &never);
        for (int k = segk - 2 > 0 ? segk - 2 : 0; k < segk; ++k) mbar_wait(&qfull[k & 1], (k >> 1) & 1, &never);
        return;
    }

    // ================= consumer warps =================
    // requests with no tokens: out = 0
    for (int b = blockIdx.x; b < p.B; b += p.num_ctas) {
        if (clamped_len(p, b) != 0) continue;
        unsigned char *o = reinterpret_cast<unsigned char *>(p.out) + (size_t)b * p.Hq * D * E;
        for (int i = tid; i < p.Hq * D / 8; i += kConsumerWarps * 32) Elem<T>::store_zero8(o + (size_t)i * 8 * E);
    }

    const int U = p.units;
    const int tsplit = p.tsplit;
    const int split = (tsplit > 1) ? warp / U : 0;
    const int units_per_g = p.G / HC;
    float *s_sm = reinterpret_cast<float *>(smem + p.off_scratch) + warp * (2 * kSubTile * HC);
    float *p_sm = s_sm + kSubTile * HC;

    typename C::Unit unit[UPW];
    int u_g[UPW], u_h0[UPW];
#pragma unroll
    for (int k = 0; k < UPW; ++k) {
        const int uid = (tsplit > 1) ? warp % U : warp + k * kConsumerWarps;
        u_g[k] = uid / units_per_g;                            // KV head within the group
        u_h0[k] = u_g[k] * p.G + (uid % units_per_g) * HC;     // first query head within the vr
    }
    const int sl = lane % C::RL;
    const int tg = lane / C::RL;

    Seg s;
    int64_t fill = 0;
    int segk = 0;
    while (it.next(p, s)) {
        // -- q of this vr --
        const int qb = segk & 1;
        if (!*abort_flag && !mbar_wait(&qfull[qb], (segk >> 1) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(p.error, PA_DEVERR_TIMEOUT);
        }
        const unsigned char *qs = qarea + qb * p.q_bytes;
#pragma unroll
        for (int k = 0; k < UPW; ++k) {
#pragma unroll
            for (int h = 0; h < HC; ++h) {
                float2 q2[4];
                Elem<T>::load8(qs + ((size_t)(u_h0[k] + h) * D + sl * 8) * E, q2);
                const float2 sc = make_float2(p.qscale, p.qscale);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    unit[k].q2[h][i] = fmul2(q2[i], sc);
                    unit[k].o2[h][i] = make_float2(0.f, 0.f);
                }
            }
            unit[k].m_own = -INFINITY;
            unit[k].l_own = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qb]);

        // -- tiles --
        for (int t = s.t_begin; t < s.t_end; ++t) {
            const int stage = (int)(fill % S);
            if (!*abort_flag && !mbar_wait(&full[stage], (uint32_t)((fill / S) & 1), abort_flag)) {
                *abort_flag = 1;
                set_error(p.error, PA_DEVERR_TIMEOUT);
            }
            if (!*abort_flag) {
                const unsigned char *kst = stage_base + (size_t)stage * 2 * p.half_bytes;
                const unsigned char *vst = kst + p.half_bytes;
                const int ntok = min(p.ST, s.L - t * p.ST);
                for (int st = split; st * kSubTile < ntok; st += tsplit) {
                    const int nvalid = min(kSubTile, ntok - st * kSubTile);
#pragma unroll
                    for (int k = 0; k < UPW; ++k)
                        C::subtile(unit[k], kst + (size_t)st * kSubTile * p.row_bytes,
                                   vst + (size_t)st * kSubTile * p.row_bytes, u_g[k], nvalid, p.row_bytes, s_sm,
                                   p_sm, lane);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            ++fill;
        }
        ++segk;

        // -- finish the piece --
#pragma unroll
        for (int k = 0; k < UPW; ++k) C::reduce_token_groups(unit[k]);

        if (tsplit > 1) {
            // warps of split > 0 hand their state to the split-0 warp of the same unit
            float *comb = reinterpret_cast<float *>(smem + p.off_comb) + warp * kCombStride;
            if (split > 0) {
#pragma unroll
                for (int h = 0; h < HC; ++h) {
                    const float mh = __shfl_sync(0xffffffffu, unit[0].m_own, h * C::LPH);
                    const float lh = __shfl_sync(0xffffffffu, unit[0].l_own, h * C::LPH);
                    if (tg == 0) {
                        Elem<float>::store8(comb + h * D + sl * 8, unit[0].o2[h]);
                        if (sl == 0) {
                            comb[HC * D + h] = mh;
                            comb[HC * D + HC + h] = lh;
                        }
                    }
                }
            }
            named_barrier(1, kConsumerWarps * 32);
            if (split == 0) {
                for (int s2 = 1; s2 < tsplit; ++s2) {
                    const float *oc = reinterpret_cast<const float *>(smem + p.off_comb) + (warp + s2 * U) * kCombStride;
#pragma unroll
                    for (int h = 0; h < HC; ++h) {
                        const float m1 = __shfl_sync(0xffffffffu, unit[0].m_own, h * C::LPH);
                        const float l1 = __shfl_sync(0xffffffffu, unit[0].l_own, h * C::LPH);
                        const float m2 = oc[HC * D + h];
                        const float l2 = oc[HC * D + HC + h];
                        const float M = fmaxf(m1, m2);
                        const float a1 = exp2f(m1 - M), a2 = exp2f(m2 - M);
                        float2 o2[4];
                        Elem<float>::load8(oc + h * D + sl * 8, o2);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            unit[0].o2[h][i].x = unit[0].o2[h][i].x * a1 + o2[i].x * a2;
                            unit[0].o2[h][i].y = unit[0].o2[h][i].y * a1 + o2[i].y * a2;
                        }
                        if (lane / C::LPH == h) {
                            unit[0].m_own = M;
                            unit[0].l_own = l1 * a1 + l2 * a2;
                        }
                    }
                }
            }
            named_barrier(1, kConsumerWarps * 32);
        }

        const bool writer = (split == 0);
        if (s.nparts == 1) {
            if (writer && !*abort_flag) {
#pragma unroll
                for (int k = 0; k < UPW; ++k)
#pragma unroll
                    for (int h = 0; h < HC; ++h) {
                        const float lh = __shfl_sync(0xffffffffu, unit[k].l_own, h * C::LPH);
                        if (tg == 0) {
                            const float inv = 1.f / lh;
                            float2 r[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                r[i] = make_float2(unit[k].o2[h][i].x * inv, unit[k].o2[h][i].y * inv);
                            const size_t hgl = (size_t)s.hg * p.NHvr + u_h0[k] + h;
                            Elem<T>::store8(reinterpret_cast<unsigned char *>(p.out) +
                                                (((size_t)s.b * p.Hq + hgl) * D + sl * 8) * E,
                                            r);
                        }
                    }
            }
            continue;
        }

        // partial piece: leave (m, l, o) in the slot, then count arrivals
        const bool slot_ok = s.slot < p.max_slots;
        if (writer && slot_ok) {
            float *base = p.partials + s.slot * p.slot_floats;
#pragma unroll
            for (int k = 0; k < UPW; ++k)
#pragma unroll
                for (int h = 0; h < HC; ++h) {
                    const float mh = __shfl_sync(0xffffffffu, unit[k].m_own, h * C::LPH);
                    const float lh = __shfl_sync(0xffffffffu, unit[k].l_own, h * C::LPH);
                    const int hl = u_h0[k] + h;
                    if (tg == 0) {
                        Elem<float>::store8(base + (size_t)hl * D + sl * 8, unit[k].o2[h]);
                        if (sl == 0) {
                            base[p.NHvr * D + hl] = mh;
                            base[p.NHvr * D + p.NHvr + hl] = lh;
                        }
                    }
                }
        }
        if (!slot_ok && tid == 0) set_error(p.error, PA_DEVERR_WORKSPACE);
        __threadfence();
        named_barrier(1, kConsumerWarps * 32);
        const int64_t vr = (int64_t)s.b * p.NHG + s.hg;
        if (tid == 0) {
            const int prev = atomicAdd(&p.counters[vr], 1);
            ctl.merge_flag = (prev == s.nparts - 1);
        }
        named_barrier(1, kConsumerWarps * 32);
        if (ctl.merge_flag) {
            __threadfence();
            // combine every piece of this vr by log-sum-exp
            const int64_t NTc = NT;
            const int64_t c0 = cta_of(s.vr_start, NTc, Cn);
            const int nq = p.NHvr * (D / 4);
            for (int idx = tid; idx < nq; idx += kConsumerWarps * 32) {
                const int h = idx / (D / 4);
                const int d4 = idx % (D / 4);
                float M = -INFINITY;
                for (int i = 0; i < s.nparts; ++i) {
                    int64_t slot;
                    if (p.mode == PA_SPLIT_BALANCED) {
                        const int64_t c = c0 + i;
                        slot = 2 * c + (s.vr_start <= range_lo(c, NTc, Cn) ? 0 : 1);
                    } else {
                        slot = s.vr_start + i;
                    }
                    if (slot >= p.max_slots) continue;
                    const float *base = p.partials + slot * p.slot_floats;
                    M = fmaxf(M, __ldcg(base + p.NHvr * D + h));
                }
                float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
                float den = 0.f;
                for (int i = 0; i < s.nparts; ++i) {
                    int64_t slot;
                    if (p.mode == PA_SPLIT_BALANCED) {
                        const int64_t c = c0 + i;
                        slot = 2 * c + (s.vr_start <= range_lo(c, NTc, Cn) ? 0 : 1);
                    } else {
                        slot = s.vr_start + i;
                    }
                    if (slot >= p.max_slots) continue;
                    const float *base = p.partials + slot * p.slot_floats;
                    const float w = exp2f(__ldcg(base + p.NHvr * D + h) - M);
                    den += w * __ldcg(base + p.NHvr * D + p.NHvr + h);
                    const float4 o = __ldcg(reinterpret_cast<const float4 *>(base + (size_t)h * D) + d4);
                    num.x += w * o.x;
                    num.y += w * o.y;
                    num.z += w * o.z;
                    num.w += w * o.w;
                }
                const float inv = 1.f / den;
                const size_t hgl = (size_t)s.hg * p.NHvr + h;
                unsigned char *dst =
                    reinterpret_cast<unsigned char *>(p.out) + (((size_t)s.b * p.Hq + hgl) * D + d4 * 4) * E;
                if constexpr (E == 2) {
                    __nv_bfloat162 a = __floats2bfloat162_rn(num.x * inv, num.y * inv);
                    __nv_bfloat162 c = __floats2bfloat162_rn(num.z * inv, num.w * inv);
                    uint2 w2;
                    w2.x = *reinterpret_cast<uint32_t *>(&a);
                    w2.y = *reinterpret_cast<uint32_t *>(&c);
                    *reinterpret_cast<uint2 *>(dst) = w2;
                } else {
                    *reinterpret_cast<float4 *>(dst) = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
                }
            }
            if (tid == 0) p.counters[vr] = 0;
        }
    }
}

}  // namespace pa
