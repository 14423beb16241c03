// Paged decode attention for sm_100a.
//
// What it computes (BareLLM README: paged KV cache, block table, one-token
// batched decode over unequal histories; MHA/GQA/MQA): for every request b
// and query head h,
//     out[b][h] = sum_t softmax_t(scale * q[b][h] . K_t) V_t ,  t < L_b,
// where K_t / V_t is row t % bs of physical block block_tables[b][t / bs] for
// KV head h / (Hq/Hkv).  The softmax runs with a running maximum and sum
// (the online softmax of the MinivLLM review and the LLAISYS self-attention
// bullet), in fp32, in the base-2 domain (scores are scaled by scale*log2 e
// so every weight is one exp2).
//
// Work decomposition.  A "virtual request" (vr) is one request restricted to
// a group of HG KV heads (HG = Hkv unless one token of all KV heads is too
// large to stage).  Its tokens are cut into tiles of ST tokens.
//   * balanced mode: the first tiles of every vr form a static list, its last
//     share (a quarter, for batches large enough) a dynamic list.  CTA c takes
//     slice c of the static list; the dynamic list is cut into grains of about
//     an eighth of a CTA's share, handed out at run time through a global
//     counter to whichever CTA is free, so that fast and slow SMs finish
//     together.  The cut itself depends only on the lengths, so every CTA can
//     name all pieces of a vr and their partial slots.
//   * fixed mode: the units of the static list are partitions of `part_tiles`
//     tiles (the classic flash-decoding split), divided the same way; nothing
//     dynamic.  The partitions of a vr that fall in one CTA's slice are
//     combined as they stream (the online softmax carried across the
//     partition boundary is the log-sum-exp combination of the two), so a vr
//     leaves one partial per CTA it touches, not one per partition.
// A vr that lies wholly inside one piece is written straight to `out`.
// Otherwise each piece leaves (m, l, o) in its workspace slot and bumps the
// vr's counter; the CTA that arrives last combines the pieces by log-sum-exp
// and restores the counter to zero (no CTA ever waits for another).
//
// Inside a CTA: warp 8 is the producer.  It alone walks the work, publishes
// one descriptor per piece (with q) to the consumers, walks the block table (a
// window of 32 entries held in registers, the next window prefetched) and
// fills a ring of shared-memory stages with tensor-map boxes (bf16 / fp16) or
// bulk copies (fp32), completion counted on mbarriers.  Warps 0-7 consume;
// each owns (KV head, query heads) units of the vr and runs one of two
// engines over every 16 tokens:
//   * MmaEngine (bf16 / fp16): warp-level tensor-core tiles with tokens as the
//     M dimension: S^T = K Q^T (m16n8k16, K from shared memory by ldmatrix,
//     Q fragments in registers), online softmax on the accumulator
//     fragments, then O^T += V^T P^T (V by transposing ldmatrix, P moved into
//     operand layout by movmatrix).
//   * CoreEngine (fp32, or any dtype): lanes own 8-element slices of a token
//     row; packed fp32x2 FMAs form partial dots, a reduce-scatter across the
//     slice lanes finishes them, and every lane accumulates its 8 output
//     elements of all its heads.
// Warp 9 counts arrivals: after the consumers have stored a piece's partial it
// fences and bumps the vr's counter, so no consumer stalls on a global atomic.
//
// Fused step (append + decode in one launch): the piece holding a request's
// last position also writes the request's new K/V token to its cache slot, and
// the consumers overwrite that row of the staged tile with the new values
// before reading it, so the decode sees the appended token without waiting
// for the cache write.
#pragma once

#include <cstddef>
#include <type_traits>

#include "common.cuh"

namespace pa {

constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kArrivalWarp = kConsumerWarps + 1;
constexpr int kDecodeThreads = (kConsumerWarps + 2) * 32;
constexpr int kSubTile = 16;     // tokens per online-softmax update
constexpr int kPrefixCache = 512;  // requests whose static / dynamic prefix sums live in shared memory

struct DecodeParams {
    CUtensorMap tmap_k;   // bf16 path: [d, token row, head] view of the pools, 128B swizzle,
    CUtensorMap tmap_v;   // box {64, br, HG}: one block piece of one head group, head-major in smem
    CUtensorMap tmap_q;   // tensor-core (tcgen05) engine: [d, request*head] view of q, box {64, NHvr}
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    void *out;
    float *partials;      // [slots][slot_floats] fp32: o[NHvr][D], m[NHvr], l[NHvr], padding
    int32_t *counters;    // [B * NHG]
    int32_t *error;       // device error word
    int32_t *grab;        // dynamic grains handed out so far (reset by the last CTA)
    int32_t *grab_done;   // CTAs that found the dynamic list empty
    const void *k_new;    // fused step: [B, Hkv, D] new token per request
    const void *v_new;
    const int32_t *slot_mapping;  // fused step: [B] cache slot of the new token (< 0: none)
    float qscale;         // scale * log2(e)
    int32_t B, Hq, Hkv, bs, num_blocks, max_blocks;
    int32_t G, HG, NHG, NHvr;
    int32_t ST;           // tokens per tile (power of two, >= 16)
    int32_t stages;
    int32_t mode;         // PA_SPLIT_BALANCED / PA_SPLIT_FIXED
    int32_t part_tiles;   // fixed mode: tiles per partition
    int32_t num_ctas;
    int32_t tsplit;       // warps sharing one unit (token split)
    int32_t units;        // units per vr
    int32_t heads_per_unit;
    int32_t fused;        // 1: append the new tokens in this launch
    int32_t dyn_num;      // balanced mode: dynamic share of each vr, in 1/256 (0: all static)
    int64_t max_slots;
    int64_t slot_floats;  // NHvr * D + (2 * NHvr rounded up to a multiple of 4)
    uint32_t off_bar, off_q, off_stage, off_scratch, off_comb;
    uint32_t row_bytes;   // HG * D * elem: one token of the head group
    uint32_t row_pitch;   // bytes between token rows in a stage (row_bytes, or + 16 for ldmatrix)
    uint32_t half_bytes;  // ST * row_pitch (K part of a stage; V part follows)
    uint32_t q_bytes;     // NHvr * D * elem
    uint32_t comb_stride; // bytes per warp in the token-split combine area
    int32_t use_tmap;     // 1: stages are filled by tensor-map boxes (swizzled, head-major)
    int32_t br_log2;      // rows of one box = min(ST, bs) = 1 << br_log2
    int32_t bs_log2;
    int32_t st_log2;      // ST = 1 << st_log2
    int32_t spec;         // 0: no speculation; 1: speculate; 2: speculate on wrong guesses (tests)
    int32_t test_stall;   // tests: CTA 0 never fills the stages of its first piece (the bounded waits give up)
    int32_t lens_cached;  // context lengths were copied into shared memory
    int32_t split_merge;  // 1: split vrs are merged by a second grid (paged_merge_kernel), not in this one
    struct MergeRecord *records;  // split_merge: per vr, how its pieces map to partial slots
    int32_t use_qmap;     // 1: q is staged by tmap_q boxes (128-byte swizzle), one per 64-wide d-chunk
    int32_t dchunk_major; // 1: a stage is [d-chunk][token row][128 B] (tcgen05 engine, HG = 1)
};
static_assert(offsetof(DecodeParams, tmap_k) % 64 == 0 && offsetof(DecodeParams, tmap_v) % 64 == 0 &&
                  offsetof(DecodeParams, tmap_q) % 64 == 0,
              "tensor maps must be 64-byte aligned");

// ---------------------------------------------------------------------------
// element access
template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ void load8(const void *p, float2 (&v)[4]) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        v[0] = bf16x2_to_float2(w.x);
        v[1] = bf16x2_to_float2(w.y);
        v[2] = bf16x2_to_float2(w.z);
        v[3] = bf16x2_to_float2(w.w);
    }
    static __device__ __forceinline__ void store8(void *p, const float2 (&v)[4]) {
        uint4 w;
        w.x = pack_bf16x2(v[0].x, v[0].y);
        w.y = pack_bf16x2(v[1].x, v[1].y);
        w.z = pack_bf16x2(v[2].x, v[2].y);
        w.w = pack_bf16x2(v[3].x, v[3].y);
        *reinterpret_cast<uint4 *>(p) = w;
    }
    static __device__ __forceinline__ void store2(void *p, float a, float b) {
        *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(a, b);
    }
    static __device__ __forceinline__ void store1(void *p, float a) {
        *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(a);
    }
    static __device__ __forceinline__ void store_zero8(void *p) {
        *reinterpret_cast<uint4 *>(p) = make_uint4(0, 0, 0, 0);
    }
};

template <>
struct Elem<__half> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ void load8(const void *p, float2 (&v)[4]) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        v[0] = f16x2_to_float2(w.x);
        v[1] = f16x2_to_float2(w.y);
        v[2] = f16x2_to_float2(w.z);
        v[3] = f16x2_to_float2(w.w);
    }
    static __device__ __forceinline__ void store8(void *p, const float2 (&v)[4]) {
        uint4 w;
        w.x = pack_f16x2(v[0].x, v[0].y);
        w.y = pack_f16x2(v[1].x, v[1].y);
        w.z = pack_f16x2(v[2].x, v[2].y);
        w.w = pack_f16x2(v[3].x, v[3].y);
        *reinterpret_cast<uint4 *>(p) = w;
    }
    static __device__ __forceinline__ void store2(void *p, float a, float b) {
        *reinterpret_cast<uint32_t *>(p) = pack_f16x2(a, b);
    }
    static __device__ __forceinline__ void store1(void *p, float a) {
        *reinterpret_cast<__half *>(p) = __float2half_rn(a);
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
    static __device__ __forceinline__ void store2(void *p, float a, float b) {
        *reinterpret_cast<float2 *>(p) = make_float2(a, b);
    }
    static __device__ __forceinline__ void store1(void *p, float a) { *reinterpret_cast<float *>(p) = a; }
    static __device__ __forceinline__ void store_zero8(void *p) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4 *>(p)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
};

// Read every scalar launch parameter once, so that the constant cache holds
// them before the prologue's dependent chain starts.
__device__ __forceinline__ void warm_params(const DecodeParams &p) {
    asm volatile("" ::"l"(p.q), "l"(p.k_cache), "l"(p.v_cache), "l"(p.block_tables), "l"(p.context_lens),
                 "l"(p.out), "l"(p.partials), "l"(p.counters));
    asm volatile("" ::"l"(p.error), "l"(p.grab), "l"(p.grab_done), "l"(p.k_new), "l"(p.v_new), "l"(p.slot_mapping),
                 "f"(p.qscale), "l"(p.max_slots), "l"(p.slot_floats));
    asm volatile("" ::"r"(p.B), "r"(p.Hq), "r"(p.Hkv), "r"(p.bs), "r"(p.num_blocks), "r"(p.max_blocks), "r"(p.G),
                 "r"(p.HG), "r"(p.NHG), "r"(p.NHvr), "r"(p.ST), "r"(p.stages), "r"(p.mode), "r"(p.part_tiles),
                 "r"(p.num_ctas), "r"(p.tsplit), "r"(p.units), "r"(p.heads_per_unit), "r"(p.fused), "r"(p.dyn_num));
    asm volatile("" ::"r"(p.off_bar), "r"(p.off_q), "r"(p.off_stage), "r"(p.off_scratch), "r"(p.off_comb),
                 "r"(p.row_bytes), "r"(p.row_pitch), "r"(p.half_bytes), "r"(p.q_bytes), "r"(p.comb_stride),
                 "r"(p.use_tmap), "r"(p.br_log2), "r"(p.bs_log2), "r"(p.st_log2), "r"(p.spec), "r"(p.lens_cached));
}

// ---------------------------------------------------------------------------
// work list
constexpr int kLensCache = 1024;  // requests whose lengths are kept in shared memory

__device__ __forceinline__ int clamped_len(const DecodeParams &p, const int *lens_s, int b) {
    int L = p.lens_cached ? lens_s[b] : p.context_lens[b];
    const int cap = p.max_blocks * p.bs;
    return L < 0 ? 0 : (L > cap ? cap : L);
}

// work units of a request: tiles (balanced) or partitions (fixed)
__device__ __forceinline__ int units_of_len(const DecodeParams &p, int L) {
    const int tiles = (L + p.ST - 1) >> p.st_log2;
    return p.mode == PA_SPLIT_BALANCED ? tiles : (tiles + p.part_tiles - 1) / p.part_tiles;
}

// units of a vr of T units that go to the dynamic list
__device__ __forceinline__ int dyn_units(int T, int dyn_num) { return (int)(((int64_t)T * dyn_num) >> 8); }

// The cut of the work (identical in every CTA): the static list (every vr's
// first units, vr after vr) in Cn slices, and the dynamic list (every vr's
// remaining units, vr after vr) in J grains of g units.
struct Cut {
    int64_t S, Dn;  // units in the static / dynamic list
    int64_t Cn;     // CTAs with a static slice
    int64_t g, J;
    int dyn;        // the dynamic list is in use
    double inv_S, inv_Cn, inv_g;  // 1/S, 1/Cn, 1/g rounded to nearest (for floor_div_inv)
};

// (positions and products stay far below 2^52, so these quotients are exact)
__device__ __forceinline__ int64_t slice_lo(int64_t r, const Cut &k) { return floor_div_inv(r * k.S, k.Cn, k.inv_Cn); }
// static slice holding static-list position x
__device__ __forceinline__ int64_t slice_of(int64_t x, const Cut &k) {
    return floor_div_inv((x + 1) * k.Cn - 1, k.S, k.inv_S);
}

// The cut from the totals: tq units over all requests (one head group), dq of
// them dynamic.
__device__ __forceinline__ Cut make_cut(int64_t tq, int64_t dq, int NHG, int64_t C, bool may_dyn) {
    const int64_t NT = tq * NHG;
    Cut k;
    k.dyn = may_dyn && dq > 0 && NT >= 4 * C && NT < (int64_t(1) << 30);
    k.Dn = k.dyn ? dq * NHG : 0;
    k.S = NT - k.Dn;
    k.Cn = k.S < C ? (k.S > 0 ? k.S : 1) : C;
    k.g = floor_div_exact(NT + 8 * C - 1, 8 * C);
    if (k.g < 1) k.g = 1;
    k.J = k.dyn ? floor_div_exact(k.Dn + k.g - 1, k.g) : 0;
    k.inv_S = __drcp_rn((double)(k.S > 0 ? k.S : 1));
    k.inv_Cn = __drcp_rn((double)k.Cn);
    k.inv_g = __drcp_rn((double)k.g);
    return k;
}

struct Seg {
    int b, hg, L;         // b < 0: no more work
    int t_begin, t_end;   // tiles of the vr this piece covers
    int nparts;           // pieces of the vr (1: the whole vr is in this piece)
    int s_len, d_len;     // static / dynamic units of the vr
    int64_t slot;         // partial slot when nparts > 1
    int64_t ss, ds;       // list positions of the vr's first static / dynamic unit
    int32_t patch;        // fused step: vr token that is the new token (-1: none)
    int32_t append_slot;  // fused step: cache slot the new token goes to (-1: none)
};

// Pieces of a vr in balanced mode: one per static slice and one per grain its
// units fall in.  Static piece (vr v, slice r) owns slot v + r and dynamic
// piece (vr v, grain j) slot NV + C + v + j: a later vr never lies in an
// earlier slice or grain, so no two pieces share a slot.
__device__ __forceinline__ int balanced_parts(const Cut &k, int64_t ss, int s_len, int64_t ds, int d_len) {
    const int ns = (int)(slice_of(ss + s_len - 1, k) - slice_of(ss, k) + 1);
    const int nd = d_len > 0 ? (int)(floor_div_inv(ds + d_len - 1, k.g, k.inv_g) - floor_div_inv(ds, k.g, k.inv_g) + 1) : 0;
    return ns + nd;
}

// Partial slots of the pieces of a vr: piece i < ns at a + i, the others at
// b + (i - ns).
struct PieceSlots {
    int64_t a, b;
    int ns;
    __device__ __forceinline__ int64_t operator()(int i) const { return i < ns ? a + i : b + (i - ns); }
};

__device__ __forceinline__ PieceSlots piece_slots(const DecodeParams &p, const Cut &k, const Seg &s) {
    PieceSlots r;
    const int64_t v = (int64_t)s.b * p.NHG + s.hg;
    const int64_t r0 = slice_of(s.ss, k);
    r.ns = (int)(slice_of(s.ss + s.s_len - 1, k) - r0 + 1);
    r.a = v + r0;
    r.b = (int64_t)p.B * p.NHG + p.num_ctas + v + (s.d_len > 0 ? floor_div_inv(s.ds, k.g, k.inv_g) : 0);
    return r;
}

// What the merge grid needs of a vr: its pieces and their partial slots
// (PieceSlots), written each launch by the CTA holding the vr's first unit.
struct MergeRecord {
    int32_t nparts, ns;
    int64_t a, b;
};

// pieces of this CTA's static slice, in list order
struct SegIter {
    int64_t cur, hi;
    int64_t vr_start, ds;  // list positions of the current vr's first static / dynamic unit
    int b, hg, L, su, du;  // current vr: request, head group, length, static / dynamic units
    const int *lens_s;

    __device__ __forceinline__ void load_request(const DecodeParams &p, const Cut &k) {
        L = clamped_len(p, lens_s, b);
        const int T = units_of_len(p, L);
        du = k.dyn ? dyn_units(T, p.dyn_num) : 0;
        su = T - du;
    }

    __device__ __forceinline__ bool next(const DecodeParams &p, const Cut &k, Seg &s) {
        while (cur < hi) {
            if (cur >= vr_start + su) {
                vr_start += su;
                ds += du;
                if (++hg == p.NHG) {
                    hg = 0;
                    if (++b >= p.B) return false;
                    load_request(p, k);
                }
                continue;
            }
            const int u0 = (int)(cur - vr_start);
            int u1;
            s.b = b;
            s.hg = hg;
            s.L = L;
            s.s_len = su;
            s.d_len = du;
            s.ss = vr_start;
            s.ds = ds;
            s.patch = -1;
            s.append_slot = -1;
            // the run of this vr's units inside the slice is one piece
            const int64_t end = vr_start + su < hi ? vr_start + su : hi;
            u1 = (int)(end - vr_start);
            if (p.mode == PA_SPLIT_BALANCED) {
                s.t_begin = u0;
                s.t_end = u1;
            } else {
                const int tiles = (L + p.ST - 1) >> p.st_log2;
                s.t_begin = u0 * p.part_tiles;
                s.t_end = min(tiles, u1 * p.part_tiles);
            }
            s.nparts = balanced_parts(k, vr_start, su, ds, du);
            s.slot = (int64_t)b * p.NHG + hg + blockIdx.x;
            cur = vr_start + u1;
            return true;
        }
        return false;
    }
};

// pieces of grain j of the dynamic list (balanced mode, prefix sums in shared memory)
struct GrainIter {
    int64_t y, y1, j;

    __device__ __forceinline__ bool next(const DecodeParams &p, const Cut &k, const int *lens_s, const int *pre_s,
                                         const int *pre_d, Seg &s) {
        if (y >= y1) return false;
        // request holding dynamic position y: pre_d[b] <= y < pre_d[b + 1]
        int lo = 0, hi = p.B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre_d[mid] <= y) lo = mid;
            else hi = mid;
        }
        const int b = lo;
        const int L = clamped_len(p, lens_s, b);
        const int T = units_of_len(p, L);
        const int du = dyn_units(T, p.dyn_num);
        const int su = T - du;
        const int64_t off = y - pre_d[b];
        if (du <= 0 || off < 0 || off >= (int64_t)du * p.NHG) {  // inconsistent tables: stop, never index past them
            set_error(p.error, PA_DEVERR_TIMEOUT);
            y = y1;
            return false;
        }
        const int hg = (int)(off / du);
        const int w = (int)(off - (int64_t)hg * du);
        const int n = (int)(du - w < y1 - y ? du - w : y1 - y);
        s.b = b;
        s.hg = hg;
        s.L = L;
        s.t_begin = su + w;
        s.t_end = su + w + n;
        s.s_len = su;
        s.d_len = du;
        s.ss = pre_s[b] + (int64_t)hg * su;
        s.ds = pre_d[b] + (int64_t)hg * du;
        s.nparts = balanced_parts(k, s.ss, su, s.ds, du);
        s.slot = (int64_t)p.B * p.NHG + p.num_ctas + (int64_t)b * p.NHG + hg + j;
        s.patch = -1;
        s.append_slot = -1;
        y += n;
        return true;
    }
};

constexpr int kMaxPending = 16;  // split pieces a CTA holds before it merges

constexpr int kMaxWarps = 12;  // the largest CTA of any engine, in warps

struct __align__(16) DecodeCtl {
    int64_t red[kMaxWarps][2];
    Cut cut;
    int64_t found_b, found_excl, found_dexcl;
    int abort;
    Seg segs[2];               // published by the producer together with q
    Seg pending[kMaxPending];  // pieces whose partial is stored; b < 0 ends the list
    int last[kMaxPending];     // set by the arrival warp: this CTA completed the vr
    uint32_t tmem_base;        // tcgen05 engine: tensor-memory address of the CTA's allocation
};

// Barrier of the eight consumer warps on an mbarrier, so that every wait is
// bounded (a warp that gave up after a timeout cannot leave the others
// waiting for good, as a named barrier could).
struct ConsumerBarrier {
    uint64_t *bar;
    uint32_t par;
    __device__ __forceinline__ bool sync(volatile int *abort_flag, int lane) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
        const bool ok = mbar_wait(bar, par, abort_flag);
        par ^= 1u;
        return ok;
    }
};

// ---------------------------------------------------------------------------
// reduce-scatter of N per-lane values across the slice lanes (lane bits below
// log2 of the group).  Each lane stores its values in an order permuted by
// its own lane bits, so that at every step both partners keep v[0..H) and
// send v[H..2H): no selects.  Afterwards v[0..) holds value indices
// [sl*N/RL, (sl+1)*N/RL), or index sl / (RL/N) when N < RL.
template <int N, int M>
struct ReduceScatter {
    static __device__ __forceinline__ void run(float *v) {
        if constexpr (M >= 1) {
            if constexpr (N > 1) {
                constexpr int H = N / 2;
#pragma unroll
                for (int i = 0; i < H; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i + H], M);
                ReduceScatter<H, M / 2>::run(v);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
                ReduceScatter<1, M / 2>::run(v);
            }
        }
    }
};

template <int N>
struct ReduceScatter<N, 0> {
    static __device__ __forceinline__ void run(float *) {}
};

// ===========================================================================
// CUDA-core engine
// ===========================================================================
template <typename T, int D, int HC, int UPW>
struct CoreEngine {
    static constexpr int RL = D / 8;          // lanes per token row (8 elements each)
    static constexpr int TG = 32 / RL;        // token rows per warp load
    static constexpr int R = kSubTile / TG;   // rounds per sub-tile
    static constexpr int NV = R * HC;         // partial dots per lane
    static constexpr int NVL = NV >= RL ? NV / RL : 1;
    static constexpr int LPH = (32 / HC) < 16 ? (32 / HC) : 16;  // softmax lanes per head
    static constexpr int TPL = kSubTile / LPH;                   // tokens per softmax lane
    static constexpr int E = Elem<T>::kBytes;
    static constexpr bool kPaddedRows = false;
    static constexpr bool kTcgen05 = false;
    static constexpr int kThreads = kDecodeThreads;
    static constexpr bool kPairs = false;  // subtile_pair not provided
    static constexpr int kUnitsPerWarp = UPW;
    static constexpr int kCombFloats = HC * D + 8;
    static constexpr int kScratchFloats = 2 * kSubTile * HC;

    // value index = h*R + r; bits flipped per lane by the reduce-scatter order
    static constexpr int kLogR = R == 8 ? 3 : (R == 4 ? 2 : (R == 2 ? 1 : 0));
    static constexpr int kLogNV = NV >= 32 ? 5 : NV >= 16 ? 4 : NV >= 8 ? 3 : NV >= 4 ? 2 : NV >= 2 ? 1 : 0;
    static constexpr int kLogRL = RL == 16 ? 4 : 3;
    static constexpr int kScatter = kLogNV < kLogRL ? kLogNV : kLogRL;

    struct Unit {
        float2 q2[HC][4];
        float2 o2[HC][4];
        float m_own, l_own;  // running max / sum of head (lane / LPH), base-2 domain
    };

    int sl, tg, perm, head_flip, round_flip;

    __device__ __forceinline__ void setup(int lane) {
        sl = lane % RL;
        tg = lane / RL;
        perm = 0;
#pragma unroll
        for (int k = 0; k < kScatter; ++k) {
            const int lane_bit = (sl >> (kLogRL - 1 - k)) & 1;
            perm |= lane_bit << (kLogNV - 1 - k);
        }
        head_flip = perm >> kLogR;
        round_flip = perm & (R - 1);
    }

    __device__ __forceinline__ void init_unit(Unit &u, const unsigned char *qs, int h0, float qscale) const {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            float2 q2[4];
            Elem<T>::load8(qs + ((size_t)(h0 + (h ^ head_flip)) * D + sl * 8) * E, q2);
            const float2 sc = make_float2(qscale, qscale);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                u.q2[h][i] = fmul2(q2[i], sc);
                u.o2[h][i] = make_float2(0.f, 0.f);
            }
        }
        u.m_own = -INFINITY;
        u.l_own = 0.f;
    }

    __device__ __forceinline__ void subtile(Unit &u, const unsigned char *tile_k, const unsigned char *tile_v, int st,
                                            int g_local, int nvalid, const DecodeParams &p, float *s_sm, float *p_sm,
                                            int lane) const {
        const uint32_t pitch = p.row_pitch;
        const unsigned char *kst = tile_k + (size_t)st * kSubTile * pitch;
        const unsigned char *vst = tile_v + (size_t)st * kSubTile * pitch;
        const uint32_t col = (uint32_t)(g_local * D + sl * 8) * E;

        // ---- QK: partial dots over this lane's 8 elements (rounds permuted per lane) ----
        float acc[NV];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int tok = (r ^ round_flip) * TG + tg;
            float2 k2[4];
            if (tok < nvalid) {
                Elem<T>::load8(kst + tok * pitch + col, k2);
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
        ReduceScatter<NV, RL / 2>::run(acc);
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int i = (NV >= RL) ? sl * NVL + j : sl / (RL / NV);
            const int h = i / R, r = i % R;
            s_sm[h * kSubTile + r * TG + tg] = acc[j];
        }
        __syncwarp();

        // ---- online softmax per head ----
        const int hs = lane / LPH;
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
        const float alpha = exp2f(u.m_own - m_new);
        float psum = 0.f;
#pragma unroll
        for (int k = 0; k < TPL; ++k) {
            const float pk = exp2f(sc[k] - m_new);
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
                Elem<T>::load8(vst + tok * pitch + col, v2);
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

    // running max / sum of head h, broadcast to every lane
    __device__ __forceinline__ float head_m(const Unit &u, int h) const { return __shfl_sync(0xffffffffu, u.m_own, h * LPH); }
    __device__ __forceinline__ float head_l(const Unit &u, int h) const { return __shfl_sync(0xffffffffu, u.l_own, h * LPH); }

    // sum the output partials of the TG token-groups (lanes with equal slice)
    __device__ __forceinline__ void finish_unit(Unit &u) const {
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

    // hand the unit's state to another warp of the same unit (token split)
    __device__ __forceinline__ void save(const Unit &u, float *comb, int lane) const {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            const float mh = head_m(u, h), lh = head_l(u, h);
            if (tg == 0) {
                Elem<float>::store8(comb + h * D + sl * 8, u.o2[h]);
                if (sl == 0) {
                    comb[HC * D + h] = mh;
                    comb[HC * D + HC + h] = lh;
                }
            }
        }
    }

    __device__ __forceinline__ void absorb(Unit &u, const float *oc, int lane) const {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            const float m1 = head_m(u, h), l1 = head_l(u, h);
            const float m2 = oc[HC * D + h], l2 = oc[HC * D + HC + h];
            const float M = fmaxf(m1, m2);
            const float a1 = exp2f(m1 - M), a2 = exp2f(m2 - M);
            float2 o2[4];
            Elem<float>::load8(oc + h * D + sl * 8, o2);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                u.o2[h][i].x = u.o2[h][i].x * a1 + o2[i].x * a2;
                u.o2[h][i].y = u.o2[h][i].y * a1 + o2[i].y * a2;
            }
            if (lane / LPH == h) {
                u.m_own = M;
                u.l_own = l1 * a1 + l2 * a2;
            }
        }
    }

    // normalised output of the unit's heads (h_out0 = first head's index in out)
    __device__ __forceinline__ void write_out(const Unit &u, unsigned char *outb, size_t h_out0) const {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            const float lh = head_l(u, h);
            if (tg == 0) {
                const float inv = 1.f / lh;
                float2 r[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) r[i] = make_float2(u.o2[h][i].x * inv, u.o2[h][i].y * inv);
                Elem<T>::store8(outb + ((h_out0 + h) * D + sl * 8) * E, r);
            }
        }
    }

    __device__ __forceinline__ void write_partial(const Unit &u, float *slot, int NHvr, int hl0) const {
#pragma unroll
        for (int h = 0; h < HC; ++h) {
            const float mh = head_m(u, h), lh = head_l(u, h);
            if (tg == 0) {
                Elem<float>::store8(slot + (size_t)(hl0 + h) * D + sl * 8, u.o2[h]);
                if (sl == 0) {
                    slot[NHvr * D + hl0 + h] = mh;
                    slot[NHvr * D + NHvr + hl0 + h] = lh;
                }
            }
        }
    }
};

// ===========================================================================
// tensor-core engine (bf16 / fp16): tokens are the M dimension of every tile.
// PAIR: the instantiation for units whose subtiles are split between warps
// (large head groups), which steps through two full subtiles at a time.
// ===========================================================================
template <typename T, int D, int UPW, bool PAIR = false>
struct MmaEngine {
    using Op = Mma16<T>;
    static constexpr int KS = D / 16;  // k-steps of QK (over d) = m-tiles of PV (over d)
    static constexpr int E = 2;
    static constexpr bool kPaddedRows = true;
    static constexpr bool kTcgen05 = false;
    static constexpr int kThreads = kDecodeThreads;
    static constexpr bool kPairs = PAIR;  // subtile_pair: two full subtiles in one online-softmax step
    static constexpr int kUnitsPerWarp = UPW;
    static constexpr int kCombFloats = 4 * KS * 32 + 4 * 32;  // fragment-ordered o, then m, l
    static constexpr int kScratchFloats = 0;

    struct Unit {
        uint32_t qb[KS][2];  // B fragments of Q: head g4, d pairs
        float o[KS][4];      // O^T: rows d = mt*16 + g4 (+8), cols heads 2*t4, 2*t4+1
        float m[2], l[2];    // heads 2*t4, 2*t4+1 of the unit, base-2 domain
    };

    int g4, t4;
    int a_tok, a_col;  // this lane's ldmatrix row for QK (K tile)
    int v_tok, v_col;  // and for PV (V tile, transposed load)
    float qscale;
    int nreal;         // real heads in a unit (<= 8)

    __device__ __forceinline__ void setup(int lane) {
        g4 = lane >> 2;
        t4 = lane & 3;
        a_tok = (lane & 7) + ((lane >> 3) & 1) * 8;
        a_col = (lane >> 4) * 8;
        v_tok = (lane & 7) + ((lane >> 4) & 1) * 8;
        v_col = ((lane >> 3) & 1) * 8;
    }

    __device__ __forceinline__ void init_unit(Unit &u, const unsigned char *qs, int h0, float qs_) {
        qscale = qs_;
        // head g4 of the unit (rows past the real heads are zero)
        const bool real = g4 < nreal;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(qs + (size_t)(h0 + g4) * D * E);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            u.qb[ks][0] = real ? qrow[ks * 8 + t4] : 0u;
            u.qb[ks][1] = real ? qrow[ks * 8 + 4 + t4] : 0u;
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) u.o[mt][i] = 0.f;
        u.m[0] = u.m[1] = -INFINITY;
        u.l[0] = u.l[1] = 0.f;
    }

    // Stage layout (filled by tensor-map boxes): [piece][d-chunk of 64][head][row][128 B],
    // each 128-byte row stored with the 128B swizzle (16-byte chunk c of row r at c ^ (r & 7)).
    // Address of 16-byte chunk `cid` (0..15 over the head's D) of row `tok` of the tile.
    static __device__ __forceinline__ const unsigned char *row_ptr(const unsigned char *tile, int tok, int g_local,
                                                                  const DecodeParams &p) {
        const int piece = tok >> p.br_log2, r = tok & ((1 << p.br_log2) - 1);
        const uint32_t head_bytes = 128u << p.br_log2;
        return tile + ((size_t)piece * (D / 64) * p.HG + g_local) * head_bytes + r * 128;
    }
    static __device__ __forceinline__ uint32_t chunk_off(int cid, int swz, const DecodeParams &p) {
        // d-chunk (cid / 8) selects the 64-element half; within it the swizzled 16-byte slot
        return (uint32_t)(cid >> 3) * ((uint32_t)p.HG << (7 + p.br_log2)) + (uint32_t)(((cid & 7) ^ swz) << 4);
    }

    __device__ __forceinline__ void subtile(Unit &u, const unsigned char *tile_k, unsigned char *tile_v, int st,
                                            int g_local, int nvalid, const DecodeParams &p, float *, float *,
                                            int lane) const {
        // ---- S^T[16 tok x 8 heads] = K Q^T (two accumulation chains) ----
        float s[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const unsigned char *ka = row_ptr(tile_k, st * kSubTile + a_tok, g_local, p);
        const int swz = a_tok & 7;
#pragma unroll
        for (int ks = 0; ks < KS; ks += 2) {
            uint32_t a[4], b[4];
            ldmatrix_x4(a, ka + chunk_off(ks * 2 + (a_col >> 3), swz, p));
            ldmatrix_x4(b, ka + chunk_off((ks + 1) * 2 + (a_col >> 3), swz, p));
            Op::mma(s, a, u.qb[ks][0], u.qb[ks][1]);
            Op::mma(sb, b, u.qb[ks + 1][0], u.qb[ks + 1][1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] += sb[i];
        // ---- online softmax over the 16 tokens, per head column ----
        const bool v0 = g4 < nvalid, v1 = g4 + 8 < nvalid;
        const float s0 = v0 ? s[0] * qscale : -INFINITY;
        const float s1 = v0 ? s[1] * qscale : -INFINITY;
        const float s2 = v1 ? s[2] * qscale : -INFINITY;
        const float s3 = v1 ? s[3] * qscale : -INFINITY;
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
        }
        const float mn0 = fmaxf(u.m[0], mx0), mn1 = fmaxf(u.m[1], mx1);
        const float al0 = exp2_fast(u.m[0] - mn0), al1 = exp2_fast(u.m[1] - mn1);
        const float p0 = exp2_fast(s0 - mn0), p1 = exp2_fast(s1 - mn1);  // token g4
        const float p2 = exp2_fast(s2 - mn0), p3 = exp2_fast(s3 - mn1);  // token g4 + 8
        float r0 = p0 + p2, r1 = p1 + p3;
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            r0 += __shfl_xor_sync(0xffffffffu, r0, m);
            r1 += __shfl_xor_sync(0xffffffffu, r1, m);
        }
        u.l[0] = u.l[0] * al0 + r0;
        u.l[1] = u.l[1] * al1 + r1;
        u.m[0] = mn0;
        u.m[1] = mn1;
        // P = hi + lo, both bf16: the PV product then carries ~16 bits of each
        // weight instead of 8 (one bf16 P alone misses the tolerance on very
        // short, peaked contexts)
        const uint32_t ph0 = Op::pack_p(p0, p1), ph1 = Op::pack_p(p2, p3);
        const float2 h0 = Op::unpack(ph0), h1 = Op::unpack(ph1);
        const uint32_t pl0 = Op::pack_p(p0 - h0.x, p1 - h0.y), pl1 = Op::pack_p(p2 - h1.x, p3 - h1.y);
        // P^T fragments (k = token, n = head)
        const uint32_t bh0 = movmatrix_trans(ph0), bh1 = movmatrix_trans(ph1);
        const uint32_t bl0 = movmatrix_trans(pl0), bl1 = movmatrix_trans(pl1);
        if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                u.o[mt][0] *= al0;
                u.o[mt][1] *= al1;
                u.o[mt][2] *= al0;
                u.o[mt][3] *= al1;
            }
        }
        // rows past nvalid may hold stale data: zero this head's rows there
        if (nvalid < kSubTile) {
            for (int i = lane; i < (kSubTile - nvalid) * (D / 8); i += 32) {
                const int tok = st * kSubTile + nvalid + i / (D / 8);
                const int cid = i % (D / 8);
                unsigned char *row = const_cast<unsigned char *>(row_ptr(tile_v, tok, g_local, p));
                *reinterpret_cast<uint4 *>(row + chunk_off(cid, 0, p)) = make_uint4(0, 0, 0, 0);
            }
            fence_async_smem();  // ordered before the next tensor-map fill of this stage
            __syncwarp();
        }
        // ---- O^T[d x heads] += V^T P^T ----
        const unsigned char *va = row_ptr(tile_v, st * kSubTile + v_tok, g_local, p);
        const int vswz = v_tok & 7;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            uint32_t a[4];
            ldmatrix_x4_trans(a, va + chunk_off(mt * 2 + (v_col >> 3), vswz, p));
            Op::mma(u.o[mt], a, bh0, bh1);
            Op::mma(u.o[mt], a, bl0, bl1);
        }
    }

    // Two full subtiles (sa, sb: 32 tokens, no row past the context) in one
    // online-softmax step: both S^T products as four independent chains, one
    // maximum / rescale / sum over the 32 tokens, then both O^T updates.  The
    // result is that of two subtile() calls (one softmax step over a longer
    // run of tokens), with twice the independent work between the waits.
    __device__ __forceinline__ void subtile_pair(Unit &u, const unsigned char *tile_k, const unsigned char *tile_v,
                                                 int sa, int sb, int g_local, const DecodeParams &p) const {
        float s[2][4] = {}, t[2][4] = {};
        const unsigned char *ka0 = row_ptr(tile_k, sa * kSubTile + a_tok, g_local, p);
        const unsigned char *ka1 = row_ptr(tile_k, sb * kSubTile + a_tok, g_local, p);
        const int swz = a_tok & 7;
#pragma unroll
        for (int ks = 0; ks < KS; ks += 2) {
            uint32_t a0[4], b0[4], a1[4], b1[4];
            ldmatrix_x4(a0, ka0 + chunk_off(ks * 2 + (a_col >> 3), swz, p));
            ldmatrix_x4(a1, ka1 + chunk_off(ks * 2 + (a_col >> 3), swz, p));
            ldmatrix_x4(b0, ka0 + chunk_off((ks + 1) * 2 + (a_col >> 3), swz, p));
            ldmatrix_x4(b1, ka1 + chunk_off((ks + 1) * 2 + (a_col >> 3), swz, p));
            Op::mma(s[0], a0, u.qb[ks][0], u.qb[ks][1]);
            Op::mma(s[1], a1, u.qb[ks][0], u.qb[ks][1]);
            Op::mma(t[0], b0, u.qb[ks + 1][0], u.qb[ks + 1][1]);
            Op::mma(t[1], b1, u.qb[ks + 1][0], u.qb[ks + 1][1]);
        }
        float x[2][4];
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) x[k][i] = (s[k][i] + t[k][i]) * qscale;
        // head 2*t4 uses elements 0, 2 (tokens g4, g4 + 8); head 2*t4+1 uses 1, 3
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
        float mx1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
        }
        const float mn0 = fmaxf(u.m[0], mx0), mn1 = fmaxf(u.m[1], mx1);
        const float al0 = exp2_fast(u.m[0] - mn0), al1 = exp2_fast(u.m[1] - mn1);
        float pr[2][4];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            pr[k][0] = exp2_fast(x[k][0] - mn0);
            pr[k][1] = exp2_fast(x[k][1] - mn1);
            pr[k][2] = exp2_fast(x[k][2] - mn0);
            pr[k][3] = exp2_fast(x[k][3] - mn1);
        }
        float r0 = (pr[0][0] + pr[0][2]) + (pr[1][0] + pr[1][2]);
        float r1 = (pr[0][1] + pr[0][3]) + (pr[1][1] + pr[1][3]);
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            r0 += __shfl_xor_sync(0xffffffffu, r0, m);
            r1 += __shfl_xor_sync(0xffffffffu, r1, m);
        }
        u.l[0] = u.l[0] * al0 + r0;
        u.l[1] = u.l[1] * al1 + r1;
        u.m[0] = mn0;
        u.m[1] = mn1;
        // P^T fragments (k = token, n = head), high and low 16-bit parts, per subtile
        uint32_t bh[2][2], bl[2][2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint32_t ph0 = Op::pack_p(pr[k][0], pr[k][1]), ph1 = Op::pack_p(pr[k][2], pr[k][3]);
            const float2 h0 = Op::unpack(ph0), h1 = Op::unpack(ph1);
            const uint32_t pl0 = Op::pack_p(pr[k][0] - h0.x, pr[k][1] - h0.y);
            const uint32_t pl1 = Op::pack_p(pr[k][2] - h1.x, pr[k][3] - h1.y);
            bh[k][0] = movmatrix_trans(ph0);
            bh[k][1] = movmatrix_trans(ph1);
            bl[k][0] = movmatrix_trans(pl0);
            bl[k][1] = movmatrix_trans(pl1);
        }
        if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                u.o[mt][0] *= al0;
                u.o[mt][1] *= al1;
                u.o[mt][2] *= al0;
                u.o[mt][3] *= al1;
            }
        }
        // ---- O^T[d x heads] += V^T P^T over both subtiles ----
        const unsigned char *va0 = row_ptr(tile_v, sa * kSubTile + v_tok, g_local, p);
        const unsigned char *va1 = row_ptr(tile_v, sb * kSubTile + v_tok, g_local, p);
        const int vswz = v_tok & 7;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            uint32_t a0[4], a1[4];
            ldmatrix_x4_trans(a0, va0 + chunk_off(mt * 2 + (v_col >> 3), vswz, p));
            ldmatrix_x4_trans(a1, va1 + chunk_off(mt * 2 + (v_col >> 3), vswz, p));
            Op::mma(u.o[mt], a0, bh[0][0], bh[0][1]);
            Op::mma(u.o[mt], a1, bh[1][0], bh[1][1]);
            Op::mma(u.o[mt], a0, bl[0][0], bl[0][1]);
            Op::mma(u.o[mt], a1, bl[1][0], bl[1][1]);
        }
    }

    __device__ __forceinline__ void finish_unit(Unit &) const {}

    __device__ __forceinline__ void save(const Unit &u, float *comb, int lane) const {
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) comb[(mt * 4 + i) * 32 + lane] = u.o[mt][i];
        comb[(4 * KS + 0) * 32 + lane] = u.m[0];
        comb[(4 * KS + 1) * 32 + lane] = u.m[1];
        comb[(4 * KS + 2) * 32 + lane] = u.l[0];
        comb[(4 * KS + 3) * 32 + lane] = u.l[1];
    }

    __device__ __forceinline__ void absorb(Unit &u, const float *oc, int lane) const {
        float a1[2], a2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float m2 = oc[(4 * KS + j) * 32 + lane], l2 = oc[(4 * KS + 2 + j) * 32 + lane];
            const float M = fmaxf(u.m[j], m2);
            a1[j] = exp2f(u.m[j] - M);
            a2[j] = exp2f(m2 - M);
            u.l[j] = u.l[j] * a1[j] + l2 * a2[j];
            u.m[j] = M;
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                u.o[mt][i] = u.o[mt][i] * a1[i & 1] + oc[(mt * 4 + i) * 32 + lane] * a2[i & 1];
    }

    __device__ __forceinline__ void write_out(const Unit &u, unsigned char *outb, size_t h_out0) const {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int h = 2 * t4 + j;
            if (h >= nreal) continue;
            const float inv = 1.f / u.l[j];
            unsigned char *row = outb + (h_out0 + h) * D * E;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                Elem<T>::store1(row + (mt * 16 + g4) * E, u.o[mt][j] * inv);
                Elem<T>::store1(row + (mt * 16 + g4 + 8) * E, u.o[mt][2 + j] * inv);
            }
        }
    }

    __device__ __forceinline__ void write_partial(const Unit &u, float *slot, int NHvr, int hl0) const {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int h = 2 * t4 + j;
            if (h >= nreal) continue;
            float *row = slot + (size_t)(hl0 + h) * D;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                row[mt * 16 + g4] = u.o[mt][j];
                row[mt * 16 + g4 + 8] = u.o[mt][2 + j];
            }
            if (g4 == 0) {
                slot[NHvr * D + hl0 + h] = u.m[j];
                slot[NHvr * D + NHvr + hl0 + h] = u.l[j];
            }
        }
    }
};

// ===========================================================================
// producer warp
// ===========================================================================

// Wait (bounded: twice the pipeline limit) until another warp of the CTA has
// given up and raised the abort flag.
__device__ __forceinline__ void wait_for_abort(const volatile int *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (!*abort_flag && globaltimer_ns() - t0 < 2 * kWaitLimitNs) __nanosleep(100000);
}

struct ProducerState {
    int stage = 0;
    uint32_t phase = 0;
    int qslot = 0;
    uint32_t qphase = 0;
    uint32_t issued = 0, issued_par = 0;  // per stage: filled at least once / parity of the last fill
    bool ok = true;
    bool grab_issued = false;
    int grab_val = 0;  // lane 0: result of the pending grab
};

// The block-table entries a piece reads, 32 at a time: lane i holds entry
// base + i of the current window, and the next window is loaded one window
// ahead.  In the first window (where prefix-cached blocks sit) nb_val holds
// the following request's entry in the same column: a block both rows name
// (a prefix block the next request shares) is worth keeping in L2 until that
// request reads it.
struct TableWindow {
    const int32_t *table;
    const int32_t *next_table;  // the following request's row (nullptr: none)
    int nblk, next_nblk;
    int cur_base, cur_val, nxt_base, nxt_val, nb_val;

    __device__ __forceinline__ int next_row(int col) const {
        return (next_table && col < 32 && col < next_nblk) ? next_table[col] : -2;
    }
    // load the window holding the piece's first tile (and the one after it)
    __device__ __forceinline__ void prime(const DecodeParams &p, const Seg &s, const int *lens_s, int lane) {
        table = p.block_tables + (size_t)s.b * p.max_blocks;
        nblk = (s.L + p.bs - 1) >> p.bs_log2;
        next_table = s.b + 1 < p.B ? table + p.max_blocks : nullptr;
        next_nblk = next_table ? (clamped_len(p, lens_s, s.b + 1) + p.bs - 1) >> p.bs_log2 : 0;
        cur_base = ((s.t_begin * p.ST) >> p.bs_log2) & ~31;
        nxt_base = cur_base + 32;
        cur_val = (cur_base + lane < nblk) ? table[cur_base + lane] : -1;
        nxt_val = (nxt_base + lane < nblk) ? table[nxt_base + lane] : -1;
        nb_val = next_row(cur_base + lane);
    }
    // make the window holding block-table column jb current
    __device__ __forceinline__ void advance(int jb, int lane) {
        const int wb = jb & ~31;
        if (wb == cur_base) return;
        if (wb == nxt_base) {
            cur_val = nxt_val;
        } else {
            cur_val = (wb + lane < nblk) ? table[wb + lane] : -1;
        }
        cur_base = wb;
        nxt_base = wb + 32;
        nxt_val = (nxt_base + lane < nblk) ? table[nxt_base + lane] : -1;  // one window ahead
        nb_val = next_row(wb + lane);
    }
};

// Fused step: if this piece holds the vr's last token, find where the new
// token goes.  It is patched into the staged tile only when its slot is the
// request's own last position; any other slot is reported.
__device__ __forceinline__ void fused_info(const DecodeParams &p, Seg &s, int lane) {
    if (!p.fused || s.t_end != (s.L + p.ST - 1) >> p.st_log2) return;
    int sm = -1, expect = -1;
    if (lane == 0) {
        sm = p.slot_mapping[s.b];
        const int t = s.L - 1;
        const int phys = p.block_tables[(size_t)s.b * p.max_blocks + (t >> p.bs_log2)];
        expect = (phys >= 0 && phys < p.num_blocks) ? phys * p.bs + (t & (p.bs - 1)) : -1;
    }
    sm = __shfl_sync(0xffffffffu, sm, 0);
    expect = __shfl_sync(0xffffffffu, expect, 0);
    if (sm < 0) return;
    if ((int64_t)sm >= (int64_t)p.num_blocks * p.bs) {
        if (lane == 0) set_error(p.error, PA_DEVERR_SLOT);
        return;
    }
    s.append_slot = sm;
    if (sm == expect) s.patch = s.L - 1;
    else if (lane == 0) set_error(p.error, PA_DEVERR_SLOT);
}

// Hand a piece (or the end marker, b < 0) and its q to the consumers.
__device__ __forceinline__ void publish(const DecodeParams &p, ProducerState &ps, const Seg &s, DecodeCtl &ctl,
                                        uint64_t *qfull, uint64_t *qempty, unsigned char *qarea,
                                        volatile int *abort_flag, int D, int E, int lane) {
    if (!mbar_wait(&qempty[ps.qslot], ps.qphase ^ 1u, abort_flag)) {
        ps.ok = false;
        return;
    }
    if (lane == 0) {
        ctl.segs[ps.qslot] = s;
        if (s.b >= 0) {
            mbar_arrive_expect_tx(&qfull[ps.qslot], p.q_bytes);
            if (p.use_qmap) {
                // [d-chunk][head][128 B], 128-byte swizzle: the K-major layout of the S product's B operand
                const int32_t row = s.b * p.Hq + s.hg * p.NHvr;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(qarea + ps.qslot * p.q_bytes + (size_t)c * p.NHvr * 128, &p.tmap_q, c * 64, row,
                                &qfull[ps.qslot], policy_evict_first());
            } else {
                const unsigned char *qg = reinterpret_cast<const unsigned char *>(p.q);
                bulk_g2s(qarea + ps.qslot * p.q_bytes, qg + ((size_t)s.b * p.Hq + (size_t)s.hg * p.NHvr) * D * E,
                         p.q_bytes, &qfull[ps.qslot]);
            }
        } else {
            mbar_arrive(&qfull[ps.qslot]);
        }
    }
    __syncwarp();
    ps.qslot ^= 1;
    if (ps.qslot == 0) ps.qphase ^= 1u;
}

// Fill one stage per tile t_lo..t_hi-1 of the piece.  With `grab_at_last`, the
// next grain is requested while the piece's last tile is being issued.
template <int D, int E>
__device__ __forceinline__ void issue_tiles(const DecodeParams &p, ProducerState &ps, const Seg &s, int t_lo,
                                            int t_hi, TableWindow &win, bool grab_at_last, uint64_t *full,
                                            uint64_t *empty, unsigned char *stage_base, volatile int *abort_flag,
                                            uint64_t policy, uint64_t policy_keep, int lane) {
    const unsigned char *kc = reinterpret_cast<const unsigned char *>(p.k_cache);
    const unsigned char *vc = reinterpret_cast<const unsigned char *>(p.v_cache);
    const uint32_t row_bytes = p.row_bytes, pitch = p.row_pitch;
    const size_t tok_stride = (size_t)p.Hkv * D * E;  // bytes between token rows in the pool
    const bool contiguous = (p.HG == p.Hkv) && (pitch == row_bytes);
    for (int t = t_lo; t < t_hi; ++t) {
        if (!mbar_wait(&empty[ps.stage], ps.phase ^ 1u, abort_flag)) {
            ps.ok = false;
            return;
        }
        if (grab_at_last && t == s.t_end - 1 && !ps.grab_issued) {
            if (lane == 0) ps.grab_val = atomicAdd(p.grab, 1);
            ps.grab_issued = true;
        }
        const int tok0 = t * p.ST;
        const int ntok = min(p.ST, s.L - tok0);
        const int jb0 = tok0 >> p.bs_log2;
        win.advance(jb0, lane);
        const int cur_base = win.cur_base, cur_val = win.cur_val, nb_val = win.nb_val;
        unsigned char *kdst = stage_base + (size_t)ps.stage * 2 * p.half_bytes;
        unsigned char *vdst = kdst + p.half_bytes;
        uint32_t bytes = 0;
        if (p.use_tmap) {
            // one box {64 d, br rows, HG heads} per (block piece, 64-wide d-chunk), for K and V
            const int br = 1 << p.br_log2;
            const int npc = (ntok + br - 1) >> p.br_log2;  // pieces holding valid tokens
            const uint32_t box_bytes = (uint32_t)p.HG << (7 + p.br_log2);
            constexpr int NDC = D / 64;
            const int tp = tok0 + lane * br;  // first token of this lane's piece
            const int j = tp >> p.bs_log2;
            const int phys = __shfl_sync(0xffffffffu, cur_val, (j - cur_base) & 31);
            const int next_phys = __shfl_sync(0xffffffffu, nb_val, (j - cur_base) & 31);
            const uint64_t pol = next_phys == phys ? policy_keep : policy;
            bool valid = false;
            if (lane < npc) {
                valid = phys >= 0 && phys < p.num_blocks;
                if (!valid) set_error(p.error, PA_DEVERR_BLOCK_ID);
                else bytes = 2u * NDC * box_bytes;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
            if (lane == 0) mbar_arrive_expect_tx(&full[ps.stage], bytes);
            __syncwarp();
            if (valid) {
                const int32_t row = phys * p.bs + (tp & (p.bs - 1));
                const int32_t head0 = s.hg * p.HG;
#pragma unroll
                for (int c2 = 0; c2 < NDC; ++c2) {
                    // head-major stage: [piece][d-chunk][head][row]; d-chunk-major: [d-chunk][token row]
                    const size_t off = p.dchunk_major ? (size_t)c2 * p.ST * 128 + (size_t)lane * box_bytes
                                                      : (size_t)(lane * NDC + c2) * box_bytes;
                    tma_load_3d(kdst + off, &p.tmap_k, c2 * 64, row, head0, &full[ps.stage], pol);
                    tma_load_3d(vdst + off, &p.tmap_v, c2 * 64, row, head0, &full[ps.stage], pol);
                }
            }
        } else if (contiguous) {
            // one copy per block piece: rows of all KV heads are contiguous in both places
            const int np = ((tok0 + ntok - 1) >> p.bs_log2) - jb0 + 1;
            const int j = jb0 + lane;
            const int phys = __shfl_sync(0xffffffffu, cur_val, (j - cur_base) & 31);
            int tlo = 0, nrows = 0;
            bool valid = false;
            if (lane < np) {
                tlo = max(tok0, j * p.bs);
                nrows = min(tok0 + ntok, (j + 1) * p.bs) - tlo;
                valid = phys >= 0 && phys < p.num_blocks;
                if (!valid) set_error(p.error, PA_DEVERR_BLOCK_ID);
                else bytes = 2u * (uint32_t)nrows * row_bytes;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
            if (lane == 0) mbar_arrive_expect_tx(&full[ps.stage], bytes);
            __syncwarp();
            if (valid) {
                const size_t src = ((size_t)phys * p.bs + (tlo - j * p.bs)) * tok_stride;
                const uint32_t n = (uint32_t)nrows * row_bytes;
                bulk_g2s_hint(kdst + (tlo - tok0) * pitch, kc + src, n, &full[ps.stage], policy);
                bulk_g2s_hint(vdst + (tlo - tok0) * pitch, vc + src, n, &full[ps.stage], policy);
            }
        } else {
            // one copy per token row (a head group narrower than the pool row)
            for (int i0 = 0; i0 < ntok; i0 += 32) {
                const int i = i0 + lane;
                const int tt = tok0 + i;
                const int j = tt >> p.bs_log2;
                const int phys = __shfl_sync(0xffffffffu, cur_val, (j - cur_base) & 31);
                if (i < ntok) {
                    if (phys < 0 || phys >= p.num_blocks) set_error(p.error, PA_DEVERR_BLOCK_ID);
                    else bytes += 2u * row_bytes;
                }
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
            if (lane == 0) mbar_arrive_expect_tx(&full[ps.stage], bytes);
            __syncwarp();
            for (int i0 = 0; i0 < ntok; i0 += 32) {
                const int i = i0 + lane;
                const int tt = tok0 + i;
                const int j = tt >> p.bs_log2;
                const int phys = __shfl_sync(0xffffffffu, cur_val, (j - cur_base) & 31);
                if (i < ntok && phys >= 0 && phys < p.num_blocks) {
                    const size_t src = ((size_t)phys * p.bs + (tt - j * p.bs)) * tok_stride + (size_t)s.hg * row_bytes;
                    bulk_g2s_hint(kdst + i * pitch, kc + src, row_bytes, &full[ps.stage], policy);
                    bulk_g2s_hint(vdst + i * pitch, vc + src, row_bytes, &full[ps.stage], policy);
                }
            }
        }
        ps.issued |= 1u << ps.stage;
        ps.issued_par = (ps.issued_par & ~(1u << ps.stage)) | (ps.phase << ps.stage);
        if (++ps.stage == p.stages) {
            ps.stage = 0;
            ps.phase ^= 1u;
        }
    }
}

template <int D, int E>
__device__ __forceinline__ void run_producer(const DecodeParams &p, const Cut &k, SegIter it, DecodeCtl &ctl,
                                             const int *lens_s, const int *pre_s, const int *pre_d, uint64_t *full,
                                             uint64_t *empty, uint64_t *qfull, uint64_t *qempty,
                                             unsigned char *qarea, unsigned char *stage_base,
                                             volatile int *abort_flag, int lane) {
    const uint64_t policy = policy_evict_first();        // K/V read once per step
    const uint64_t policy_keep = policy_evict_normal();  // blocks the next request shares
    ProducerState ps;
    Seg s;
    TableWindow win;
    // this CTA's static slice
    while (ps.ok && it.next(p, k, s)) {
        win.prime(p, s, lens_s, lane);  // in flight while q is published
        fused_info(p, s, lane);
        if (p.split_merge && s.t_begin == 0 && lane == 0) {
            // the vr's first unit: record how its pieces map to slots for the merge grid
            const PieceSlots sl = piece_slots(p, k, s);
            MergeRecord r;
            r.nparts = s.nparts;
            r.ns = sl.ns;
            r.a = sl.a;
            r.b = sl.b;
            p.records[(int64_t)s.b * p.NHG + s.hg] = r;
        }
        publish(p, ps, s, ctl, qfull, qempty, qarea, abort_flag, D, E, lane);
        if (!ps.ok) break;
        if (p.test_stall && blockIdx.x == 0) {
            // failure-path test: no stage of this piece is ever filled, so the
            // consumers' wait gives up; issue nothing and leave once they abort
            wait_for_abort(abort_flag);
            ps.ok = false;
            break;
        }
        issue_tiles<D, E>(p, ps, s, s.t_begin, s.t_end, win, k.dyn && it.cur >= it.hi, full, empty, stage_base,
                          abort_flag, policy, policy_keep, lane);
    }
    // grains of the dynamic list, one at a time, to whichever CTA asks first
    if (k.dyn) {
        for (;;) {
            if (!ps.grab_issued && lane == 0) ps.grab_val = atomicAdd(p.grab, 1);
            const int64_t j = __shfl_sync(0xffffffffu, ps.grab_val, 0);
            ps.grab_issued = false;
            if (j >= k.J) break;
            GrainIter gi;
            gi.j = j;
            gi.y = j * k.g;
            gi.y1 = gi.y + k.g < k.Dn ? gi.y + k.g : k.Dn;
            while (ps.ok && gi.next(p, k, lens_s, pre_s, pre_d, s)) {
                win.prime(p, s, lens_s, lane);
                fused_info(p, s, lane);
                publish(p, ps, s, ctl, qfull, qempty, qarea, abort_flag, D, E, lane);
                if (!ps.ok) break;
                issue_tiles<D, E>(p, ps, s, s.t_begin, s.t_end, win, gi.y >= gi.y1, full, empty, stage_base,
                                  abort_flag, policy, policy_keep, lane);
            }
        }
        // the last CTA to find the list empty leaves the counters at zero for the next launch
        if (lane == 0) {
            const int d = atomicAdd(p.grab_done, 1);
            if (d == p.num_ctas - 1) {
                atomicExch(p.grab, 0);
                atomicExch(p.grab_done, 0);
            }
        }
    }
    if (ps.ok) {
        Seg end;
        end.b = -1;
        publish(p, ps, end, ctl, qfull, qempty, qarea, abort_flag, D, E, lane);
    }
    if (!ps.ok) {
        *abort_flag = 1;
        if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
    }
    // every copy this warp issued lands before the CTA can retire
    volatile int never = 0;
    for (int st = 0; st < p.stages; ++st)
        if (ps.issued & (1u << st)) mbar_wait(&full[st], (ps.issued_par >> st) & 1u, &never);
}

// ===========================================================================
// merge of a split vr by log-sum-exp (run by the consumer warps of the CTA
// that delivered the last piece):
//     out[h] = sum_i 2^(m_i[h] - M[h]) o_i[h] / sum_i 2^(m_i[h] - M[h]) l_i[h],
//     M[h] = max_i m_i[h]  (base-2 domain; pieces with m = -inf contribute 0).
// ===========================================================================

// The pieces a merge combines: k -> the k-th piece of the list (first + k * stride
// in PieceSlots order).
struct MergeList {
    PieceSlots slots;
    int first, stride, n;
    __device__ __forceinline__ int64_t operator()(int k) const { return slots(first + k * stride); }
};

// Where a merge writes: into `out` (normalised, dtype of the cache), or into
// partial slot `slot` as (o, m, l) like a piece.
struct MergeDst {
    bool to_slot;
    int64_t slot;
    size_t out_head0;  // first head of the vr in out
};

// From registers: one pass per output element keeps a running maximum, so any
// number of pieces is combined with eight pieces' loads (o, m, l) in flight.
// Writing into a slot that is also an input (a group's first piece), every
// thread's reads come first: o elements are read and written by the same
// thread, and (m, l) are written after a barrier of the consumer warps.
template <typename T, int D>
__device__ __forceinline__ bool merge_parts(const DecodeParams &p, const MergeList &L, const MergeDst &dst, int tid,
                                            ConsumerBarrier &cb, volatile int *abort_flag) {
    constexpr int E = Elem<T>::kBytes;
    constexpr int NTH = kConsumerWarps * 32;
    constexpr int KF = 8;  // pieces per batch of loads
    const int NH = p.NHvr;
    const int nparts = L.n;
    const int nq = NH * (D / 4);
    for (int idx0 = tid; idx0 < nq; idx0 += 2 * NTH) {
        constexpr int IT = 2;  // output items per thread per batch
        int hh[IT], dd[IT];
        bool act[IT];
        float M[IT], den[IT];
        float4 num[IT];
#pragma unroll
        for (int j = 0; j < IT; ++j) {
            const int idx = idx0 + j * NTH;
            act[j] = idx < nq;
            hh[j] = act[j] ? idx / (D / 4) : 0;
            dd[j] = act[j] ? idx % (D / 4) : 0;
            M[j] = -INFINITY;
            den[j] = 0.f;
            num[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int i0 = 0; i0 < nparts; i0 += KF) {
            int64_t sl[KF];
#pragma unroll
            for (int k = 0; k < KF; ++k) {
                const int i = i0 + k;
                int64_t slot = -1;
                if (i < nparts) {
                    slot = L(i);
                    if (slot < 0 || slot >= p.max_slots) slot = -1;
                }
                sl[k] = slot;
            }
            float4 o[IT][KF];
            float mi[IT][KF], li[IT][KF];
#pragma unroll
            for (int j = 0; j < IT; ++j)
#pragma unroll
                for (int k = 0; k < KF; ++k) {
                    if (act[j] && sl[k] >= 0) {
                        const float *base = p.partials + sl[k] * p.slot_floats;
                        o[j][k] = __ldcg(reinterpret_cast<const float4 *>(base + (size_t)hh[j] * D) + dd[j]);
                        mi[j][k] = __ldcg(base + NH * D + hh[j]);
                        li[j][k] = __ldcg(base + NH * D + NH + hh[j]);
                    } else {
                        o[j][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                        mi[j][k] = -INFINITY;
                        li[j][k] = 0.f;
                    }
                }
#pragma unroll
            for (int j = 0; j < IT; ++j) {
                float cm = M[j];
#pragma unroll
                for (int k = 0; k < KF; ++k) cm = fmaxf(cm, mi[j][k]);
                if (cm == -INFINITY) continue;
                const float a = exp2f(M[j] - cm);  // M = -inf before the first piece: 0
                num[j].x *= a;
                num[j].y *= a;
                num[j].z *= a;
                num[j].w *= a;
                den[j] *= a;
#pragma unroll
                for (int k = 0; k < KF; ++k) {
                    const float w = exp2f(mi[j][k] - cm);  // missing pieces: exp2(-inf) = 0
                    den[j] += w * li[j][k];
                    num[j].x += w * o[j][k].x;
                    num[j].y += w * o[j][k].y;
                    num[j].z += w * o[j][k].z;
                    num[j].w += w * o[j][k].w;
                }
                M[j] = cm;
            }
        }
#pragma unroll
        for (int j = 0; j < IT; ++j) {
            if (!act[j]) continue;
            if (dst.to_slot) {
                float *base = p.partials + dst.slot * p.slot_floats;
                reinterpret_cast<float4 *>(base + (size_t)hh[j] * D)[dd[j]] = num[j];
            } else {
                const float inv = 1.f / den[j];
                unsigned char *o8 =
                    reinterpret_cast<unsigned char *>(p.out) + ((dst.out_head0 + hh[j]) * D + dd[j] * 4) * E;
                Elem<T>::store2(o8, num[j].x * inv, num[j].y * inv);
                Elem<T>::store2(o8 + 2 * E, num[j].z * inv, num[j].w * inv);
            }
        }
    }
    if (!dst.to_slot) return true;
    // (m, l) of the merged piece, once every thread has read the inputs' (m, l):
    // per head the same maximum over the pieces the o elements were scaled by
    const bool ok = cb.sync(abort_flag, tid & 31);
    if (ok) {
        float *base = p.partials + dst.slot * p.slot_floats;
        for (int hh = tid; hh < NH; hh += NTH) {
            float M = -INFINITY;
            for (int k = 0; k < nparts; ++k) {
                const int64_t slot = L(k);
                if (slot >= 0 && slot < p.max_slots) M = fmaxf(M, __ldcg(p.partials + slot * p.slot_floats + NH * D + hh));
            }
            float den = 0.f;
            for (int k = 0; k < nparts; ++k) {
                const int64_t slot = L(k);
                if (slot < 0 || slot >= p.max_slots) continue;
                const float *b = p.partials + slot * p.slot_floats + NH * D;
                if (b[hh] != -INFINITY) den += exp2f(b[hh] - M) * __ldcg(b + NH + hh);
            }
            base[NH * D + hh] = M;
            base[NH * D + NH + hh] = den;
        }
    }
    return ok;
}

// The same merge streamed through shared memory, for a CTA's final merges
// (its pipeline stages are free by then):
//   * a ring of up to kMergeRing buffers of one piece's o block each is kept
//     filled by bulk asynchronous copies (one mbarrier per buffer), the first
//     ones issued before anything else, so that about kMergeRing copies are
//     in flight for the whole merge;
//   * meanwhile every piece's (m, l) of every head is loaded; per head the
//     maximum M and the weights w_i = 2^(m_i - M) (divided by
//     sum_j 2^(m_j - M) l_j when the merge writes `out`), each thread taking
//     every (NTH/NH)-th piece of one head;
//   * each thread adds w_i o_i to its output elements as the buffers land;
//     the last warp to finish with a buffer refills it with a later piece (a
//     shared-memory counter per buffer), so no warp waits for another.
// One exponential per (head, piece), and the merge runs at the copy rate of
// one SM instead of one round trip per batch of pieces.  The query heads of a
// vr are a power of two <= 128, so they divide the consumer threads.  Every
// consumer thread calls it; `ring` holds the ring's mbarriers and `ring_par`
// their phases (bit b: buffer b).  Returns false if a wait gave up.
constexpr int kMergeRing = 12;

template <int NTH>
__host__ __device__ constexpr size_t staged_merge_head_bytes(int nparts, int NH) {
    // weights and (m, l) [nparts][NH] x 2, two [NTH] reduction rows, the ring's counters
    return ((size_t)2 * nparts * NH * 4 + 2 * NTH * 4 + kMergeRing * 4 + 1023) & ~(size_t)1023;
}

template <typename T, int D>
__device__ __forceinline__ bool merge_parts_staged(const DecodeParams &p, const MergeList &L, const MergeDst &dst,
                                                   int tid, unsigned char *buf, uint32_t buf_bytes, uint64_t *ring,
                                                   uint32_t &ring_par, volatile int *abort_flag, ConsumerBarrier &cb) {
    constexpr int E = Elem<T>::kBytes;
    constexpr int NTH = kConsumerWarps * 32;
    constexpr int kMaxItems = 8;  // (head, 4 d) items per thread: NHvr * D <= 8192
    const int NH = p.NHvr;
    const int nparts = L.n;
    const int lane = tid & 31;
    const uint32_t o_bytes = (uint32_t)NH * D * 4u;
    const uint32_t o_off = (uint32_t)staged_merge_head_bytes<NTH>(nparts, NH);
    int nb = o_off < buf_bytes ? (int)((buf_bytes - o_off) / o_bytes) : 0;
    nb = min(min(nb, kMergeRing), nparts);
    float *w_s = reinterpret_cast<float *>(buf);  // [nparts][NH]: m, then the weights
    float *l_s = w_s + (size_t)nparts * NH;      // [nparts][NH]
    float *red = l_s + (size_t)nparts * NH;      // [2][NTH]
    int *cnt = reinterpret_cast<int *>(red + 2 * NTH);  // [kMergeRing] warps done with each buffer
    const int nq = NH * (D / 4);
    auto issue = [&](int i, int b) {  // piece i into buffer b (one thread)
        const int64_t slot = L(i);
        const bool valid = slot >= 0 && slot < p.max_slots;
        if (valid) {
            mbar_arrive_expect_tx(&ring[b], o_bytes);
            bulk_g2s(buf + o_off + (size_t)b * o_bytes, p.partials + slot * p.slot_floats, o_bytes, &ring[b]);
        } else {
            mbar_arrive(&ring[b]);  // nothing to copy: the buffer is read as weight 0
        }
    };
    // ---- the first copies, in flight while the weights are worked out ----
    if (tid == 0) {
        fence_async_smem();  // earlier reads and writes of buf before the copies overwrite it
        for (int b = 0; b < nb; ++b) {
            cnt[b] = 0;
            issue(b, b);
        }
    }
    // ---- the weights ----
    for (int x = tid; x < nparts * NH; x += NTH) {
        const int i = x / NH, h = x - (x / NH) * NH;
        const int64_t slot = L(i);
        const bool valid = slot >= 0 && slot < p.max_slots;
        const float *base = p.partials + (valid ? slot : 0) * p.slot_floats;
        w_s[x] = valid ? __ldcg(base + (size_t)NH * D + h) : -INFINITY;
        l_s[x] = valid ? __ldcg(base + (size_t)NH * D + NH + h) : 0.f;
    }
    const int h = tid & (NH - 1), sub = tid / NH, nsub = NTH / NH;
    bool ok = cb.sync(abort_flag, lane);
    float mloc = -INFINITY;
    for (int i = sub; i < nparts; i += nsub) mloc = fmaxf(mloc, w_s[i * NH + h]);
    red[tid] = mloc;
    if (!cb.sync(abort_flag, lane)) ok = false;
    float M = -INFINITY;
    for (int k = 0; k < nsub; ++k) M = fmaxf(M, red[k * NH + h]);
    float dloc = 0.f;
    for (int i = sub; i < nparts; i += nsub) {
        const float m = w_s[i * NH + h];
        const float w = m == -INFINITY ? 0.f : exp2_fast(m - M);  // pieces with no token: weight 0
        w_s[i * NH + h] = (L(i) >= 0 && L(i) < p.max_slots) ? w : 0.f;
        dloc += w * l_s[i * NH + h];
    }
    red[NTH + tid] = dloc;
    if (!cb.sync(abort_flag, lane)) ok = false;
    float den = 0.f;
    for (int k = 0; k < nsub; ++k) den += red[NTH + k * NH + h];
    if (!dst.to_slot) {
        const float inv = 1.f / den;
        for (int i = sub; i < nparts; i += nsub) w_s[i * NH + h] *= inv;
    }
    if (!cb.sync(abort_flag, lane)) ok = false;
    // ---- sum_i w_i o_i as the buffers land ----
    float4 acc[kMaxItems];
#pragma unroll
    for (int j = 0; j < kMaxItems; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < nparts && ok; ++i) {
        const int b = i % nb;
        if (!mbar_wait(&ring[b], (ring_par >> b) & 1u, abort_flag)) {
            ok = false;
            break;
        }
        ring_par ^= 1u << b;
        const float4 *ob = reinterpret_cast<const float4 *>(buf + o_off + (size_t)b * o_bytes);
        const float *wi = w_s + (size_t)i * NH;
        const bool filled = L(i) >= 0 && L(i) < p.max_slots;  // else the buffer holds nothing of piece i
#pragma unroll
        for (int j = 0; j < kMaxItems; ++j) {
            const int idx = tid + j * NTH;
            if (idx < nq && filled) {
                const float w = wi[idx / (D / 4)];
                const float4 o = ob[idx];  // o[h][d] at h * D + d: float4 index h * (D/4) + d/4 = idx
                acc[j].x += w * o.x;
                acc[j].y += w * o.y;
                acc[j].z += w * o.z;
                acc[j].w += w * o.w;
            }
        }
        // the last warp done with buffer b refills it with piece i + nb
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            const int done = atomicAdd(&cnt[b], 1);
            if (done == kConsumerWarps - 1) {
                __threadfence_block();
                cnt[b] = 0;
                if (i + nb < nparts) {
                    fence_async_smem();
                    issue(i + nb, b);
                }
            }
        }
    }
    if (!ok && tid == 0) {
        // a wait gave up: let every copy still in flight into the ring land before
        // the stages are left (bounded; a buffer with no copy pending times out)
        volatile int never = 0;
        for (int b = 0; b < nb; ++b) mbar_wait(&ring[b], (ring_par >> b) & 1u, &never);
    }
    // every buffer's last copy has been waited for by every thread
    if (!cb.sync(abort_flag, lane)) ok = false;
    if (ok) {
        if (dst.to_slot) {
            // a partial: o unnormalised (relative to M), then M and the sum
            float *base = p.partials + dst.slot * p.slot_floats;
#pragma unroll
            for (int j = 0; j < kMaxItems; ++j) {
                const int idx = tid + j * NTH;
                if (idx < nq) reinterpret_cast<float4 *>(base)[idx] = acc[j];
            }
            if (sub == 0) {
                base[NH * D + h] = M;
                base[NH * D + NH + h] = den;
            }
        } else {
            const size_t out0 = dst.out_head0 * D;
#pragma unroll
            for (int j = 0; j < kMaxItems; ++j) {
                const int idx = tid + j * NTH;
                if (idx < nq) {
                    unsigned char *o8 = reinterpret_cast<unsigned char *>(p.out) + (out0 + (size_t)idx * 4) * E;
                    Elem<T>::store2(o8, acc[j].x, acc[j].y);
                    Elem<T>::store2(o8 + 2 * E, acc[j].z, acc[j].w);
                }
            }
        }
    }
    return ok;
}

// One merge: streamed through the stages when allowed and worth it (more
// pieces than two batches of register loads), else from registers.
template <typename T, int D>
__device__ __forceinline__ bool merge_run(const DecodeParams &p, const MergeList &L, const MergeDst &dst, int tid,
                                          ConsumerBarrier &cb, volatile int *abort_flag, unsigned char *stage_area,
                                          uint32_t stage_bytes, uint64_t *ring, uint32_t &ring_par) {
    const size_t need = staged_merge_head_bytes<kConsumerWarps * 32>(L.n, p.NHvr) + (size_t)2 * p.NHvr * D * 4;
    if (stage_area != nullptr && L.n > 16 && need <= stage_bytes)
        return merge_parts_staged<T, D>(p, L, dst, tid, stage_area, stage_bytes, ring, ring_par, abort_flag, cb);
    return merge_parts<T, D>(p, L, dst, tid, cb, abort_flag);
}

// Merge every vr for which this CTA delivered the last piece.  The arrival
// warp has counted the arrivals of pieces [0, npend) and signals `adone`
// once it has; its counting atomics acquire what the other pieces' CTAs
// released, so their partials are visible to the loads below.  `more`: more
// pieces follow, so the pending list is handed back afterwards.  The final
// call (`more` false) finds the pipeline stages free and may stream the merge
// through them (`stage_area`, `stage_bytes`, the ring mbarriers `ring`).
template <typename T, int D>
__device__ __forceinline__ bool flush_pending(const DecodeParams &p, DecodeCtl &ctl, int npend, uint64_t *adone,
                                              uint32_t adone_par, volatile int *abort_flag, ConsumerBarrier &cb,
                                              bool more, int tid, unsigned char *stage_area = nullptr,
                                              uint32_t stage_bytes = 0, uint64_t *ring = nullptr) {
    bool ok = mbar_wait(adone, adone_par, abort_flag);
    if (ok) {
        const Cut cut = ctl.cut;
        unsigned char *area = more ? nullptr : stage_area;
        uint32_t ring_par = 0;
        // the streamed merge needs every consumer past its tiles (true once adone
        // has completed for the final list) and its generic accesses to the
        // stages ordered before the bulk copies
        if (area) {
            fence_async_smem();
            if (!cb.sync(abort_flag, tid & 31)) ok = false;
        }
        for (int k = 0; k < npend && ok; ++k) {
            if (!ctl.last[k]) continue;
            const Seg sk = ctl.pending[k];
            const MergeDst to_out{false, 0, (size_t)sk.b * p.Hq + (size_t)sk.hg * p.NHvr};
            ok = merge_run<T, D>(p, MergeList{piece_slots(p, cut, sk), 0, 1, sk.nparts}, to_out, tid, cb, abort_flag,
                                 area, stage_bytes, ring, ring_par);
            if (tid == 0) p.counters[(int64_t)sk.b * p.NHG + sk.hg] = 0;
            if (area && !cb.sync(abort_flag, tid & 31)) ok = false;  // the stages are free for the next merge
        }
    }
    if (!ok) {
        *abort_flag = 1;
        if (tid == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
    }
    if (more) cb.sync(abort_flag, tid & 31);  // pending list free again
    return ok;
}

// Arrival warp: for each stored piece, in order, fence and count it on the
// vr's counter; the piece that completes the vr is marked for merging.
__device__ __forceinline__ void run_arrivals(const DecodeParams &p, DecodeCtl &ctl, uint64_t *pdone, uint64_t *adone,
                                             volatile int *abort_flag, int lane) {
    uint32_t pdone_par = 0;  // bit k: parity of pdone[k]'s next phase
    int k = 0;
    for (;;) {
        if (!mbar_wait(&pdone[k], (pdone_par >> k) & 1u, abort_flag)) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
            return;
        }
        pdone_par ^= 1u << k;
        const Seg s = ctl.pending[k];
        if (s.b < 0) break;
        if (lane == 0) {
            // release: the consumers' partial stores, seen through pdone, before the
            // count; acquire: every other piece's partial before the merge reads them
            const int prev = atomic_add_acq_rel(&p.counters[(int64_t)s.b * p.NHG + s.hg], 1);
            ctl.last[k] = prev == s.nparts - 1;
        }
        __syncwarp();
        if (++k == kMaxPending) {
            if (lane == 0) mbar_arrive(adone);
            k = 0;
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(adone);
}

// ===========================================================================
// the fused step's new token, one KV head: lane i holds 16-byte chunks
// i, i + 32, ... of [K row | V row]
template <int D, int E>
__device__ __forceinline__ unsigned char *stage_chunk(unsigned char *tile, int tok, int g_local, int c,
                                                      const DecodeParams &p) {
    if (p.dchunk_major) {
        // [d-chunk][token row][128 B] (one KV head), 16-byte slots swizzled by row
        const int c2 = c >> 3, cc = c & 7;
        return tile + (size_t)c2 * p.ST * 128 + (size_t)tok * 128 + ((cc ^ (tok & 7)) << 4);
    }
    if (p.use_tmap) {
        // [piece][d-chunk][head][row][128 B], 16-byte slots swizzled by row
        const int piece = tok >> p.br_log2, r = tok & ((1 << p.br_log2) - 1);
        const uint32_t head_bytes = 128u << p.br_log2;
        const int c2 = c >> 3, cc = c & 7;
        return tile + ((size_t)(piece * (D / 64) + c2) * p.HG + g_local) * head_bytes + r * 128 +
               ((cc ^ (r & 7)) << 4);
    }
    return tile + (size_t)tok * p.row_pitch + (size_t)g_local * D * E + c * 16;
}

template <int D, int E>
struct NewToken {
    static constexpr int CH = D * E / 16;           // 16-byte chunks in one head's row
    static constexpr int NCH = (2 * CH + 31) / 32;  // chunks per lane
    uint4 v[NCH];

    __device__ __forceinline__ void load(const DecodeParams &p, int b, int head, int lane) {
        const size_t base = ((size_t)b * p.Hkv + head) * D * E;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane + 32 * i;
            if (c < 2 * CH) {
                const unsigned char *src = reinterpret_cast<const unsigned char *>(c < CH ? p.k_new : p.v_new);
                v[i] = __ldg(reinterpret_cast<const uint4 *>(src + base + (size_t)(c % CH) * 16));
            }
        }
    }
    // the append proper: the new token into its cache slot
    __device__ __forceinline__ void store(const DecodeParams &p, int slot, int head, int lane) const {
        const size_t base = ((size_t)slot * p.Hkv + head) * D * E;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane + 32 * i;
            if (c < 2 * CH) {
                unsigned char *dst = reinterpret_cast<unsigned char *>(const_cast<void *>(c < CH ? p.k_cache : p.v_cache));
                *reinterpret_cast<uint4 *>(dst + base + (size_t)(c % CH) * 16) = v[i];
            }
        }
    }
    // row `tok` of the staged tile takes the new token's values
    __device__ __forceinline__ void patch(unsigned char *tk, unsigned char *tv, int tok, int g_local,
                                          const DecodeParams &p, int lane) const {
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane + 32 * i;
            if (c < 2 * CH)
                *reinterpret_cast<uint4 *>(stage_chunk<D, E>(c < CH ? tk : tv, tok, g_local, c % CH, p)) = v[i];
        }
        fence_async_smem();  // ordered before the next tensor-map fill of this stage
        __syncwarp();
    }
};

// ===========================================================================
// prologue helpers
// ===========================================================================

// One request per thread (B <= kDecodeThreads): `raw` is request tid's
// length (any value past B).  One block-wide scan yields the totals (the
// cut), this CTA's static slice [lo, hi), each request's list positions and
// the request holding the slice's first unit (ctl.found_*, which must be -1
// on entry).  Contains one __syncthreads; the caller synchronises before
// reading ctl.
template <int NWARPS>
__device__ __forceinline__ Cut scan_requests(const DecodeParams &p, int raw, DecodeCtl &ctl, int *lens_s, int *pre_s,
                                             int *pre_d, bool may_dyn, int64_t &lo, int64_t &hi, int tid, int lane,
                                             int warp) {
    const int cap = p.max_blocks * p.bs;
    const int b = tid;
    int nu = 0, du = 0;
    if (b < p.B) {
        lens_s[b] = raw;  // B <= kDecodeThreads <= kLensCache: lens_cached
        nu = units_of_len(p, raw < 0 ? 0 : (raw > cap ? cap : raw));
        du = may_dyn ? dyn_units(nu, p.dyn_num) : 0;
    }
    int64_t xa = nu, xb = du;  // inclusive scan within the warp
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const int64_t ya = __shfl_up_sync(0xffffffffu, xa, m);
        const int64_t yb = __shfl_up_sync(0xffffffffu, xb, m);
        if (lane >= m) {
            xa += ya;
            xb += yb;
        }
    }
    if (lane == 31) {
        ctl.red[warp][0] = xa;
        ctl.red[warp][1] = xb;
    }
    __syncthreads();
    int64_t ta = 0, tb = 0, pa = 0, pb = 0;
    for (int w = 0; w < NWARPS; ++w) {
        const int64_t wa = ctl.red[w][0], wb = ctl.red[w][1];
        if (w < warp) {
            pa += wa;
            pb += wb;
        }
        ta += wa;
        tb += wb;
    }
    const Cut cut = make_cut(ta, tb, p.NHG, p.num_ctas, may_dyn);
    const bool has_slice = cut.S > 0 && blockIdx.x < cut.Cn;
    lo = has_slice ? slice_lo(blockIdx.x, cut) : 0;
    hi = has_slice ? slice_lo(blockIdx.x + 1, cut) : 0;
    // request b's first static / dynamic list positions and unit counts
    const int64_t ea = pa + xa - nu, eb = pb + xb - du;
    const int64_t es = (int64_t)p.NHG * (cut.dyn ? ea - eb : ea);
    const int64_t ed = cut.dyn ? (int64_t)p.NHG * eb : 0;
    const int64_t us = (int64_t)p.NHG * (cut.dyn ? nu - du : nu);
    if (b < p.B) {
        if (cut.dyn) {
            pre_s[b] = (int)es;
            pre_d[b] = (int)ed;
        }
        if (us > 0 && es <= lo && lo < es + us) {
            ctl.found_b = b;
            ctl.found_excl = es;
            ctl.found_dexcl = ed;
        }
    }
    if (tid == 0) {
        ctl.cut = cut;
        if (cut.dyn) {
            pre_s[p.B] = (int)cut.S;
            pre_d[p.B] = (int)cut.Dn;
        }
    }
    return cut;
}

// The iterator over this CTA's static slice [lo, hi), positioned by ctl.found_*.
__device__ __forceinline__ SegIter slice_iter(const DecodeParams &p, const DecodeCtl &ctl, const Cut &cut, int64_t lo,
                                              int64_t hi, const int *lens_s) {
    SegIter it;
    it.cur = lo;
    it.hi = hi;
    it.lens_s = lens_s;
    if (lo < hi && ctl.found_b >= 0) {
        it.b = (int)ctl.found_b;
        it.load_request(p, cut);
        it.hg = p.NHG == 1 ? 0 : (int)floor_div_exact(lo - ctl.found_excl, it.su);
        it.vr_start = ctl.found_excl + (int64_t)it.hg * it.su;
        it.ds = ctl.found_dexcl + (int64_t)it.hg * it.du;
    } else {
        it.cur = it.hi = 0;
        it.b = 0;
        it.hg = 0;
        it.L = 0;
        it.su = 0;
        it.du = 0;
        it.vr_start = 0;
        it.ds = 0;
    }
    return it;
}

// Speculative warm-up (producer warp, tensor-map path): the first blocks
// this CTA would stream with the guessed lengths (as far as kSpecBytes of K
// and V) pulled into L2.  It runs before the grid-dependency wait, on lengths
// and block-table entries the preceding grid may still change: nothing read
// here is used for the decode itself (the plan is kept only if every length
// read after the wait matches its guess, and the block tables are read again
// after the wait), and a wrong guess only costs bandwidth.
constexpr uint32_t kSpecBytes = 256u << 10;

template <int D>
__device__ __forceinline__ void prefetch_block(const DecodeParams &p, const Seg &s, int phys) {
    constexpr int NDC = D / 64;
    if (phys < 0 || phys >= p.num_blocks) return;
    const int32_t head0 = s.hg * p.HG;
    const int boxes = p.bs >> p.br_log2;  // boxes per block (tiles shorter than a block: several)
    for (int x = 0; x < boxes; ++x) {
        const int32_t row = phys * p.bs + (x << p.br_log2);
#pragma unroll
        for (int c2 = 0; c2 < NDC; ++c2) {
            tma_prefetch_3d(&p.tmap_k, c2 * 64, row, head0);
            tma_prefetch_3d(&p.tmap_v, c2 * 64, row, head0);
        }
    }
}

template <int D>
__device__ __forceinline__ void speculative_prefetch(const DecodeParams &p, const DecodeCtl &ctl, const Cut &cut,
                                                     int64_t lo, int64_t hi, const int *lens_s, int lane) {
    constexpr int E = 2;
    SegIter it = slice_iter(p, ctl, cut, lo, hi, lens_s);
    const uint32_t block_bytes = 2u * (uint32_t)p.bs * p.HG * D * E;
    int budget = (int)(kSpecBytes / block_bytes);
    budget = budget < 1 ? 1 : (budget > 32 ? 32 : budget);
    Seg s;
    while (budget > 0 && it.next(p, cut, s)) {  // one guessed table entry per lane and block
        const int jb0 = (s.t_begin * p.ST) >> p.bs_log2;
        const int jb1 = (min(s.t_end * p.ST, s.L) - 1) >> p.bs_log2;
        const int n = min(jb1 - jb0 + 1, budget);
        if (lane < n) prefetch_block<D>(p, s, ld_hint(p.block_tables + (size_t)s.b * p.max_blocks + jb0 + lane));
        budget -= n;
    }
}

// Requests with no tokens: out = 0 (the fused step still appends their new
// token).  Run by the consumer warps, requests dealt round-robin over CTAs.
template <typename T, int D>
__device__ __forceinline__ void zero_empty_requests(const DecodeParams &p, const int *lens_s, int tid) {
    constexpr int E = Elem<T>::kBytes;
    constexpr int NTH = kConsumerWarps * 32;
    for (int b = blockIdx.x; b < p.B; b += p.num_ctas) {
        if (clamped_len(p, lens_s, b) != 0) continue;
        unsigned char *o = reinterpret_cast<unsigned char *>(p.out) + (size_t)b * p.Hq * D * E;
        for (int i = tid; i < p.Hq * D / 8; i += NTH) Elem<T>::store_zero8(o + (size_t)i * 8 * E);
        if (p.fused) {
            const int sm = p.slot_mapping[b];
            if (sm >= 0 && (int64_t)sm >= (int64_t)p.num_blocks * p.bs) {
                if (tid == 0) set_error(p.error, PA_DEVERR_SLOT);
            } else if (sm >= 0) {
                const int nvec = p.Hkv * D * E / 16;
                for (int i = tid; i < 2 * nvec; i += NTH) {
                    const bool kk = i < nvec;
                    const uint4 *src = reinterpret_cast<const uint4 *>(kk ? p.k_new : p.v_new) + (size_t)b * nvec;
                    uint4 *dst = reinterpret_cast<uint4 *>(const_cast<void *>(kk ? p.k_cache : p.v_cache)) +
                                 (size_t)sm * nvec;
                    dst[i % nvec] = __ldg(src + i % nvec);
                }
            }
        }
    }
}

}  // namespace pa

// the tcgen05 consumer side (large query-head groups)
#include "decode_tc.cuh"

namespace pa {

// ===========================================================================
template <typename T, int D, class Engine>
__global__ void __launch_bounds__(Engine::kThreads, 1) paged_decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int E = Elem<T>::kBytes;
    constexpr bool kTC = Engine::kTcgen05;
    constexpr int kThreads = Engine::kThreads;
    constexpr int NWARPS = kThreads / 32;
    static_assert(NWARPS <= kMaxWarps, "control block");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ DecodeCtl ctl;
    __shared__ int lens_s[kLensCache];
    __shared__ int pre_s[kPrefixCache + 1], pre_d[kPrefixCache + 1];
    // swizzled tensor-map boxes need 1024-byte aligned destinations
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int S = p.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + S;
    uint64_t *qfull = empty + S;
    uint64_t *qempty = qfull + 2;
    uint64_t *pdone = qempty + 2;
    uint64_t *adone = pdone + kMaxPending;
    uint64_t *cbar = adone + 1;
    uint64_t *mbar = cbar + 1;  // the final merges' ring of bulk copies (kMergeRing)
    volatile int *abort_flag = &ctl.abort;
    unsigned char *qarea = smem + p.off_q;
    unsigned char *stage_base = smem + p.off_stage;

    uint64_t *tcb = mbar + kMergeRing;  // tcgen05 engine: sfull[2], pfull[2], odone[2], xchg[2][2], tdone, tfin
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            // tcgen05 engine: a stage is released by one commit after its P V product
            mbar_init(&empty[s], kTC ? 1 : kConsumerWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            // tcgen05 engine: the consumer warps and the P V warp arrive, and the S warp by a
            // commit after the piece's last S product (Q is read until then)
            mbar_init(&qempty[i], kTC ? kConsumerWarps + 2 : kConsumerWarps);
        }
        for (int i = 0; i < kMaxPending; ++i) mbar_init(&pdone[i], kConsumerWarps);
        mbar_init(adone, 1);
        mbar_init(cbar, kConsumerWarps);
        for (int i = 0; i < kMergeRing; ++i) mbar_init(&mbar[i], 1);
        if constexpr (kTC) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&tcb[i], 1);                    // sfull: S product done
                mbar_init(&tcb[2 + i], kConsumerWarps);   // pfull: P written
                mbar_init(&tcb[4 + i], 1);                // odone: P V product done
                mbar_init(&tcb[6 + i], 4);                // xchg, heads of the first half: four warps
                mbar_init(&tcb[8 + i], 4);                // xchg, heads of the second half
            }
            mbar_init(&tcb[10], kConsumerWarps);          // tdone: last tensor-memory read
            mbar_init(&tcb[11], 2);                       // tfin: every product of both issuers done
        }
        ctl.abort = 0;
        ctl.found_b = -1;
        fence_mbarrier_init();
    }
    if (warp == kProducerWarp && lane == 0 && p.use_tmap) {
        prefetch_tensormap(&p.tmap_k);
        prefetch_tensormap(&p.tmap_v);
        if (p.use_qmap) prefetch_tensormap(&p.tmap_q);
    }
    // ---- while the preceding grid may still run: nothing here reads its output ----
    // Warm the constant cache with the launch parameters, and pull the first
    // metadata reads of the prologue into L2: every CTA the lengths, and each
    // CTA its share of the block tables, q and (fused step) the new tokens.
    {
        if (tid == 0) warm_params(p);
        prefetch_l2_share(p.context_lens, (size_t)p.B * 4, tid, kThreads, 4);
        const size_t first = (size_t)blockIdx.x * kThreads + tid;
        const size_t stride = (size_t)gridDim.x * kThreads;
        prefetch_l2_share(p.block_tables, (size_t)p.B * p.max_blocks * 4, first, stride, 2);
        prefetch_l2_share(p.q, (size_t)p.B * p.Hq * D * E, first, stride, 2);
        if (p.fused) {
            prefetch_l2_share(p.slot_mapping, (size_t)p.B * 4, tid, kThreads, 4);
            prefetch_l2_share(p.k_new, (size_t)p.B * p.Hkv * D * E, first, stride, 1);
            prefetch_l2_share(p.v_new, (size_t)p.B * p.Hkv * D * E, first, stride, 1);
        }
    }
    // Speculative plan (batches of up to kDecodeThreads requests): the slice
    // this CTA would take with the lengths as they are now, and its first
    // blocks pulled into L2 while the preceding grid finishes.
    const int cap = p.max_blocks * p.bs;
    const bool may_dyn = p.mode == PA_SPLIT_BALANCED && p.dyn_num > 0 && p.B <= kPrefixCache && p.lens_cached;
    const bool one_pass = p.B <= kDecodeThreads;
    const bool speculate = one_pass && p.spec != 0;
    Cut cut;
    int64_t lo = 0, hi = 0;
    int guess = 0;
    if (speculate) {
        if (tid < p.B) guess = ld_hint(p.context_lens + tid) + (p.spec == 2 ? 1 + (tid & 1) : 0);
        cut = scan_requests<NWARPS>(p, guess, ctl, lens_s, pre_s, pre_d, may_dyn, lo, hi, tid, lane, warp);
        __syncthreads();
        if (warp == kProducerWarp && p.use_tmap) speculative_prefetch<D>(p, ctl, cut, lo, hi, lens_s, lane);
    }

    // everything below may read what the preceding grid on the stream wrote;
    // the next grid may start its own prologue as soon as SMs free up
    grid_dependency_wait();
    grid_launch_dependents();

    // ---- prologue: the cut of the work and this CTA's static slice ----
    if (one_pass) {
        // the lengths again, now that the preceding grid has completed: the
        // early plan stands only if every one is unchanged
        const int raw = tid < p.B ? p.context_lens[tid] : 0;
        if (blockIdx.x == 0 && tid < p.B && (raw < 0 || raw > cap)) set_error(p.error, PA_DEVERR_CONTEXT_LEN);
        if (!__syncthreads_and(speculate && raw == guess)) {
            if (tid == 0) ctl.found_b = -1;
            cut = scan_requests<NWARPS>(p, raw, ctl, lens_s, pre_s, pre_d, may_dyn, lo, hi, tid, lane, warp);
        }
    } else {
        // any batch size: the totals first, then the prefix sums chunk by chunk
        int64_t t_local = 0, d_local = 0;
        for (int b = tid; b < p.B; b += kThreads) {
            const int raw = p.context_lens[b];
            if (blockIdx.x == 0 && (raw < 0 || raw > cap)) set_error(p.error, PA_DEVERR_CONTEXT_LEN);
            if (p.lens_cached) lens_s[b] = raw;
            const int nu = units_of_len(p, raw < 0 ? 0 : (raw > cap ? cap : raw));
            t_local += nu;
            if (may_dyn) d_local += dyn_units(nu, p.dyn_num);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            t_local += __shfl_xor_sync(0xffffffffu, t_local, m);
            d_local += __shfl_xor_sync(0xffffffffu, d_local, m);
        }
        if (lane == 0) {
            ctl.red[warp][0] = t_local;
            ctl.red[warp][1] = d_local;
        }
        __syncthreads();
        if (tid == 0) {
            int64_t tq = 0, dq = 0;
            for (int w = 0; w < NWARPS; ++w) {
                tq += ctl.red[w][0];
                dq += ctl.red[w][1];
            }
            ctl.cut = make_cut(tq, dq, p.NHG, p.num_ctas, may_dyn);
        }
        __syncthreads();
        cut = ctl.cut;
        const bool has_slice = cut.S > 0 && blockIdx.x < cut.Cn;
        lo = has_slice ? slice_lo(blockIdx.x, cut) : 0;
        hi = has_slice ? slice_lo(blockIdx.x + 1, cut) : 0;

        // exclusive prefix sums of static / dynamic units over requests: the
        // request holding this CTA's first unit, and (dynamic list) the tables
        // the grains are located with
        if (lo < hi || cut.dyn) {
            int64_t run_s = 0, run_d = 0;
            for (int base = 0; base < p.B; base += kThreads) {
                const int b = base + tid;
                int64_t us = 0, ud = 0;
                if (b < p.B) {
                    const int nu = units_of_len(p, clamped_len(p, lens_s, b));
                    const int d = cut.dyn ? dyn_units(nu, p.dyn_num) : 0;
                    us = (int64_t)p.NHG * (nu - d);
                    ud = (int64_t)p.NHG * d;
                }
                int64_t xs = us, xd = ud;
#pragma unroll
                for (int m = 1; m < 32; m <<= 1) {
                    const int64_t ys = __shfl_up_sync(0xffffffffu, xs, m);
                    const int64_t yd = __shfl_up_sync(0xffffffffu, xd, m);
                    if (lane >= m) {
                        xs += ys;
                        xd += yd;
                    }
                }
                __syncthreads();  // ctl.red free to overwrite
                if (lane == 31) {
                    ctl.red[warp][0] = xs;
                    ctl.red[warp][1] = xd;
                }
                __syncthreads();
                int64_t bs_ = 0, bd_ = 0, cs = 0, cd = 0;
                for (int w = 0; w < NWARPS; ++w) {
                    if (w < warp) {
                        bs_ += ctl.red[w][0];
                        bd_ += ctl.red[w][1];
                    }
                    cs += ctl.red[w][0];
                    cd += ctl.red[w][1];
                }
                const int64_t es = run_s + bs_ + xs - us, ed = run_d + bd_ + xd - ud;
                if (cut.dyn && b < p.B) {
                    pre_s[b] = (int)es;
                    pre_d[b] = (int)ed;
                }
                if (us > 0 && es <= lo && lo < es + us) {
                    ctl.found_b = b;
                    ctl.found_excl = es;
                    ctl.found_dexcl = ed;
                }
                run_s += cs;
                run_d += cd;
                __syncthreads();
                if (!cut.dyn && ctl.found_b >= 0) break;
            }
            if (cut.dyn && tid == 0) {
                pre_s[p.B] = (int)cut.S;
                pre_d[p.B] = (int)cut.Dn;
            }
        }
    }
    if constexpr (kTC) {
        if (warp == kTcMmaWarp) tmem_alloc(&ctl.tmem_base, Engine::kTmemCols);
        tc_fence_before();
    }
    __syncthreads();
    if constexpr (kTC) tc_fence_after();

    const SegIter it = slice_iter(p, ctl, cut, lo, hi, lens_s);

    if (warp == kProducerWarp) {
        run_producer<D, E>(p, cut, it, ctl, lens_s, pre_s, pre_d, full, empty, qfull, qempty, qarea, stage_base,
                           abort_flag, lane);
        return;
    }
    if (warp == kArrivalWarp) {
        run_arrivals(p, ctl, pdone, adone, abort_flag, lane);
        return;
    }

    // ================= consumer warps =================
    if (warp < kConsumerWarps) zero_empty_requests<T, D>(p, lens_s, tid);
    if constexpr (kTC) {
        run_tc_consumers<T, D, Engine>(p, ctl, lens_s, full, empty, qfull, qempty, pdone, adone, cbar, mbar, tcb,
                                       qarea, stage_base, reinterpret_cast<float *>(smem + p.off_scratch),
                                       abort_flag, tid, warp, lane);
    } else {
    constexpr int UPW = Engine::kUnitsPerWarp;
    const int U = p.units;
    const int tsplit = p.tsplit;
    const int split = (tsplit > 1) ? warp / U : 0;
    const int HC = p.heads_per_unit;
    const int units_per_g = p.G / HC < 1 ? 1 : p.G / HC;
    float *s_sm = reinterpret_cast<float *>(smem + p.off_scratch) + warp * Engine::kScratchFloats;
    float *p_sm = s_sm + kSubTile * (Engine::kScratchFloats / (2 * kSubTile));

    Engine eng;
    eng.setup(lane);
    if constexpr (Engine::kPaddedRows) eng.nreal = p.G < 8 ? p.G : 8;
    typename Engine::Unit unit[UPW];
    NewToken<D, E> nt[UPW];
    int u_g[UPW], u_h0[UPW];
    bool u_writer[UPW];  // this warp stores the new token of the unit's KV head
#pragma unroll
    for (int k = 0; k < UPW; ++k) {
        const int uid = (tsplit > 1) ? warp % U : warp + k * kConsumerWarps;
        u_g[k] = uid / units_per_g;                          // KV head within the group
        u_h0[k] = u_g[k] * p.G + (uid % units_per_g) * HC;   // first query head within the vr
        u_writer[k] = split == 0 && uid % units_per_g == 0;
    }

    ConsumerBarrier cb{cbar, 0u};
    int stage = 0;
    uint32_t phase = 0;
    int qslot = 0;
    uint32_t qphase = 0;
    int npend = 0;
    uint32_t adone_par = 0;
    for (;;) {
        // -- the next piece and its q --
        if (!mbar_wait(&qfull[qslot], qphase, abort_flag)) {
            *abort_flag = 1;
            set_error(p.error, PA_DEVERR_TIMEOUT);
            break;
        }
        const Seg s = ctl.segs[qslot];
        if (s.b < 0) break;
        const unsigned char *qs = qarea + qslot * p.q_bytes;
#pragma unroll
        for (int k = 0; k < UPW; ++k) eng.init_unit(unit[k], qs, u_h0[k], p.qscale);
        if (s.append_slot >= 0) {
#pragma unroll
            for (int k = 0; k < UPW; ++k) nt[k].load(p, s.b, s.hg * p.HG + u_g[k], lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qslot]);
        qslot ^= 1;
        if (qslot == 0) qphase ^= 1u;
        const int patch_tile = s.patch >= 0 ? s.patch >> p.st_log2 : -1;
        const int patch_tok = s.patch - patch_tile * p.ST;

        // -- tiles --
        for (int t = s.t_begin; t < s.t_end; ++t) {
            if (!*abort_flag && !mbar_wait(&full[stage], phase, abort_flag)) {
                *abort_flag = 1;
                set_error(p.error, PA_DEVERR_TIMEOUT);
            }
            if (!*abort_flag) {
                unsigned char *kst = stage_base + (size_t)stage * 2 * p.half_bytes;
                unsigned char *vst = kst + p.half_bytes;
                const int ntok = min(p.ST, s.L - t * p.ST);
                int st = split;
                if constexpr (Engine::kPairs) {
                    // two full subtiles per step where a unit's subtiles are split
                    // between warps (large head groups: the MMA chain is the bound),
                    // away from the tile holding the appended token
                    if (t != patch_tile)
                        for (; (st + tsplit + 1) * kSubTile <= ntok; st += 2 * tsplit) {
#pragma unroll
                            for (int k = 0; k < UPW; ++k)
                                eng.subtile_pair(unit[k], kst, vst, st, st + tsplit, u_g[k], p);
                        }
                }
                for (; st * kSubTile < ntok; st += tsplit) {
                    const int nvalid = min(kSubTile, ntok - st * kSubTile);
                    if (t == patch_tile && st == patch_tok / kSubTile) {
#pragma unroll
                        for (int k = 0; k < UPW; ++k) nt[k].patch(kst, vst, patch_tok, u_g[k], p, lane);
                    }
#pragma unroll
                    for (int k = 0; k < UPW; ++k)
                        eng.subtile(unit[k], kst, vst, st, u_g[k], nvalid, p, s_sm, p_sm, lane);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == S) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // -- finish the piece --
#pragma unroll
        for (int k = 0; k < UPW; ++k) eng.finish_unit(unit[k]);
        if (s.append_slot >= 0 && !*abort_flag) {
#pragma unroll
            for (int k = 0; k < UPW; ++k)
                if (u_writer[k]) nt[k].store(p, s.append_slot, s.hg * p.HG + u_g[k], lane);
        }

        if (tsplit > 1) {
            // warps of split > 0 hand their state to the split-0 warp of the same unit
            float *comb = reinterpret_cast<float *>(smem + p.off_comb + warp * p.comb_stride);
            if (split > 0) eng.save(unit[0], comb, lane);
            cb.sync(abort_flag, lane);
            if (split == 0)
                for (int s2 = 1; s2 < tsplit; ++s2)
                    eng.absorb(unit[0],
                               reinterpret_cast<const float *>(smem + p.off_comb + (warp + s2 * U) * p.comb_stride),
                               lane);
            cb.sync(abort_flag, lane);
        }

        const bool writer = (split == 0);
        if (s.nparts == 1) {
            if (writer && !*abort_flag) {
                unsigned char *outb = reinterpret_cast<unsigned char *>(p.out);
#pragma unroll
                for (int k = 0; k < UPW; ++k)
                    eng.write_out(unit[k], outb, (size_t)s.b * p.Hq + (size_t)s.hg * p.NHvr + u_h0[k]);
            }
            continue;
        }

        // partial piece: leave (m, l, o) in the slot; the arrival warp counts
        // it once every consumer warp has stored its part (the merge grid
        // combines the pieces instead when split_merge is set)
        const bool slot_ok = s.slot < p.max_slots;
        if (writer && slot_ok) {
            float *base = p.partials + s.slot * p.slot_floats;
#pragma unroll
            for (int k = 0; k < UPW; ++k) eng.write_partial(unit[k], base, p.NHvr, u_h0[k]);
        }
        if (!slot_ok && tid == 0) set_error(p.error, PA_DEVERR_WORKSPACE);
        if (p.split_merge) continue;
        __syncwarp();
        if (tid == 0) ctl.pending[npend] = s;
        if (lane == 0) mbar_arrive(&pdone[npend]);
        if (++npend == kMaxPending) {
            flush_pending<T, D>(p, ctl, npend, adone, adone_par, abort_flag, cb, true, tid);
            adone_par ^= 1u;
            npend = 0;
        }
    }
    // close the list for the arrival warp, then merge what this CTA completed
    if (tid == 0) ctl.pending[npend].b = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&pdone[npend]);
    flush_pending<T, D>(p, ctl, npend, adone, adone_par, abort_flag, cb, false, tid, stage_base,
                        (uint32_t)S * 2u * p.half_bytes, mbar);
    }
}

// ===========================================================================
// The merge grid (plans with split_merge): one CTA per (vr, query head),
// launched behind the decode grid as its programmatic dependent.  The pieces
// of a vr are dealt to the CTA's eight warps (warp w takes pieces w, w+8, ...;
// lane = four consecutive d); a warp issues the loads of up to kMergeBatch of
// its pieces before it uses any, so a request split over as many as 64 CTAs
// costs one round trip to memory.  Each warp keeps a running maximum, sum and
// weighted o over its pieces, and the warps' results are combined by
// log-sum-exp:
//     out[h] = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,  M = max_i m_i
// (base-2 domain; pieces with m = -inf contribute 0).  A long request split
// over dozens of CTAs is then merged by as many CTAs as it has heads, all at
// once, instead of by the one CTA that delivered its last piece.
constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads) paged_merge_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int E = Elem<T>::kBytes;
    constexpr int NW = kMergeThreads / 32;
    __shared__ float sm_m[NW], sm_l[NW];
    __shared__ float4 sm_o[NW][D / 4];
    grid_dependency_wait();       // the decode grid's partials, records and lengths
    grid_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t cta = blockIdx.x;
    const int h = (int)(cta % p.NHvr);
    const int64_t v = cta / p.NHvr;
    const int b = (int)(v / p.NHG), hg = (int)(v % p.NHG);
    const int cap = p.max_blocks * p.bs;
    const int L = p.context_lens[b];
    if (L <= 0 || L > cap) return;  // no pieces (out already zero, or the length was flagged)
    const MergeRecord rec = p.records[v];
    const int n = rec.nparts;
    if (n <= 1) return;  // written directly by the decode grid
    const bool act = lane < D / 4;
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = warp; i0 < n; i0 += NW * kMergeBatch) {
        float mi[kMergeBatch], li[kMergeBatch];
        float4 o[kMergeBatch];
#pragma unroll
        for (int k = 0; k < kMergeBatch; ++k) {
            const int i = i0 + k * NW;
            const int64_t slot = i < rec.ns ? rec.a + i : rec.b + (i - rec.ns);
            const bool ok = i < n && slot >= 0 && slot < p.max_slots;
            if (i < n && !ok && lane == 0) set_error(p.error, PA_DEVERR_WORKSPACE);
            const float *base = p.partials + (ok ? slot : 0) * p.slot_floats;
            mi[k] = ok ? __ldcg(base + (size_t)p.NHvr * D + h) : -INFINITY;
            li[k] = ok ? __ldcg(base + (size_t)p.NHvr * D + p.NHvr + h) : 0.f;
            o[k] = (ok && act) ? __ldcg(reinterpret_cast<const float4 *>(base + (size_t)h * D) + lane)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float cm = M;
#pragma unroll
        for (int k = 0; k < kMergeBatch; ++k) cm = fmaxf(cm, mi[k]);
        if (cm == -INFINITY) continue;
        const float a = exp2f(M - cm);  // M = -inf before the first piece: 0
        num.x *= a;
        num.y *= a;
        num.z *= a;
        num.w *= a;
        den *= a;
#pragma unroll
        for (int k = 0; k < kMergeBatch; ++k) {
            const float w = exp2f(mi[k] - cm);  // missing pieces: exp2(-inf) = 0
            num.x += w * o[k].x;
            num.y += w * o[k].y;
            num.z += w * o[k].z;
            num.w += w * o[k].w;
            den += w * li[k];
        }
        M = cm;
    }
    if (lane == 0) {
        sm_m[warp] = M;
        sm_l[warp] = den;
    }
    if (act) sm_o[warp][lane] = num;
    __syncwarp();  // each warp meets the CTA barrier whole
    __syncthreads();
    if (warp != 0 || !act) return;
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, sm_m[w]);
    float dsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        if (sm_m[w] == -INFINITY) continue;
        const float c = exp2f(sm_m[w] - Mx);
        const float4 o = sm_o[w][lane];
        dsum += c * sm_l[w];
        acc.x += c * o.x;
        acc.y += c * o.y;
        acc.z += c * o.z;
        acc.w += c * o.w;
    }
    const float inv = 1.f / dsum;
    unsigned char *dst = reinterpret_cast<unsigned char *>(p.out) +
                         ((((size_t)b * p.Hq + (size_t)hg * p.NHvr + h) * D) + (size_t)lane * 4) * E;
    Elem<T>::store2(dst, acc.x * inv, acc.y * inv);
    Elem<T>::store2(dst + 2 * E, acc.z * inv, acc.w * inv);
}

}  // namespace pa
