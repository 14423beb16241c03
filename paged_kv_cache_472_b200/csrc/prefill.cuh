// Chunked prefill attention over the paged cache, for sm_100a.
//
// What it computes: request b owns rows query_start[b] .. query_start[b+1]-1
// of q and out, its n_b new tokens -- the last n_b of its context_lens[b]
// positions, whose K/V the append has already written to the cache.  New
// token j sits at position pos = L_b - n_b + j and attends causally:
//     out[row][h] = sum_{t <= pos} softmax_t(scale * q[row][h] . K_t) V_t
// with K_t / V_t row t % bs of physical block block_tables[b][t / bs] for KV
// head h / (Hq/Hkv).  This is the step before decode (the MinivLLM review's
// prefill path), read straight from the pages like the decode.
//
// Work decomposition: one CTA per (request, KV head, tile of QT new tokens).
// Its rows are the QT tokens x G query heads of that KV head (row r = token
// r / G, head r % G), at most 128, sixteen per consumer warp.  Every row of a
// CTA sees keys 0 .. pos of its own token, so the CTA streams keys
// 0 .. pos(last token) once and each warp masks the keys past its rows'
// positions.  Tiles holding the latest tokens see the most keys; the grid
// runs them first.
//
// Inside a CTA: warp 8 is the producer.  It copies the q rows into shared
// memory once and fills a ring of stages with tensor-map boxes of KT keys of
// K and V (the same [d, token row, head] view of the pool as the decode,
// 128-byte swizzle).  Warps 0-7 compute, per stage:
//   S = Q K^T       (m16n8k16 tiles: Q as the A operand from registers, K as
//                    the B operand by ldmatrix from the swizzled stage)
//   causal mask, fp32 online softmax per row in the base-2 domain,
//   O += P V        (P reused from the S accumulator fragments as the A
//                    operand, split into a high and a low 16-bit part as in
//                    the decode; V as the B operand by transposing ldmatrix).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace pa {

constexpr int kPrefillConsumerWarps = 8;
constexpr int kPrefillThreads = (kPrefillConsumerWarps + 1) * 32;
constexpr int kPrefillRows = kPrefillConsumerWarps * 16;  // rows per CTA (tokens x heads)

struct PrefillParams {
    CUtensorMap tmap_k;  // box {64 d, br rows, 1 head} on [d, token row, head] views of the pools
    CUtensorMap tmap_v;
    const void *q;       // [T, Hq, D]
    void *out;           // [T, Hq, D]
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *query_start;
    int32_t *error;      // device error word or nullptr
    float qscale;        // scale * log2(e)
    int32_t B, Hq, Hkv, G, bs, bs_log2, num_blocks, max_blocks;
    int32_t QT;          // new tokens per CTA (QT * G <= kPrefillRows)
    int32_t KT, kt_log2; // keys per stage
    int32_t br_log2;     // rows of one box = min(KT, bs)
    int32_t stages;
    int32_t num_qtiles;  // tiles of QT tokens the grid covers per request
    uint32_t off_q, off_stage, half_bytes;  // shared-memory layout (from the 1024-aligned base)
};
static_assert(offsetof(PrefillParams, tmap_k) % 64 == 0 && offsetof(PrefillParams, tmap_v) % 64 == 0,
              "tensor maps must be 64-byte aligned");

// Address of the 16-byte chunk holding d-columns 8*cid .. 8*cid+7 of key row
// `tok` of a stage filled by {64 d, br rows, 1 head} boxes: [piece][d-chunk of
// 64][row][128 B], each 128-byte row swizzled (chunk c of row r at c ^ (r & 7)).
template <int D>
__device__ __forceinline__ unsigned char *kv_chunk(unsigned char *tile, int tok, int cid, int br_log2) {
    constexpr int NDC = D / 64;
    const int piece = tok >> br_log2, r = tok & ((1 << br_log2) - 1);
    const uint32_t box = 128u << br_log2;  // one {64 d, br rows} box
    return tile + ((size_t)piece * NDC + (cid >> 3)) * box + (uint32_t)r * 128u +
           ((uint32_t)((cid & 7) ^ (r & 7)) << 4);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1) paged_prefill_kernel(const __grid_constant__ PrefillParams p) {
    using Op = Mma16<T>;
    constexpr int E = 2;
    constexpr int KS = D / 16;   // k-steps of S over d
    constexpr int NDC = D / 64;  // 64-wide d-chunks (one box each)
    constexpr int NO = D / 8;    // n-tiles of O over d
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ uint64_t bars[2 * 8 + 1];
    __shared__ volatile int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.stages;
    uint64_t *full = bars, *empty = bars + 8, *qbar = bars + 16;
    volatile int *abort_flag = &abort_s;

    // ---- the tile: request, KV head, new tokens [t0, t0 + ntok) ----
    const int b = blockIdx.z, g = blockIdx.y;
    const int qt = p.num_qtiles - 1 - (int)blockIdx.x;  // latest (heaviest) tiles first
    const int cap = p.max_blocks * p.bs;
    const int L = p.context_lens[b];
    const int q0 = p.query_start[b];
    const int n = p.query_start[b + 1] - q0;
    if (L < 0 || L > cap || n < 0 || n > L || n > p.num_qtiles * p.QT) {
        if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) set_error(p.error, PA_DEVERR_CONTEXT_LEN);
        return;
    }
    const int t0 = qt * p.QT;
    if (t0 >= n) return;
    const int ntok = min(p.QT, n - t0);
    const int pos0 = L - n + t0;       // position of the tile's first token
    const int kend = pos0 + ntok;      // keys 0 .. kend-1 are visible to some row
    const int ntiles = (kend + p.KT - 1) >> p.kt_log2;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kPrefillConsumerWarps);
        }
        mbar_init(qbar, 1);
        abort_s = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    unsigned char *qs = smem + p.off_q;
    unsigned char *stage_base = smem + p.off_stage;

    if (warp == kPrefillConsumerWarps) {
        // ================= producer =================
        const uint64_t policy = policy_evict_normal();  // K/V are read by every q-tile of the request
        if (lane == 0) {
            // q rows of the tile: token i, heads g*G .. g*G+G-1 are G*D contiguous elements
            const uint32_t row_bytes = (uint32_t)p.G * D * E;
            mbar_arrive_expect_tx(qbar, (uint32_t)ntok * row_bytes);
            const unsigned char *qg = static_cast<const unsigned char *>(p.q);
            for (int i = 0; i < ntok; ++i)
                bulk_g2s(qs + (size_t)i * row_bytes,
                         qg + (((size_t)(q0 + t0 + i)) * p.Hq + (size_t)g * p.G) * D * E, row_bytes, qbar);
        }
        const int32_t *table = p.block_tables + (size_t)b * p.max_blocks;
        const int br = 1 << p.br_log2;
        const uint32_t box_bytes = 128u << p.br_log2;
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int kt = 0; kt < ntiles && ok; ++kt) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            const int k0 = kt * p.KT;
            const int nk = min(p.KT, kend - k0);
            const int npc = (nk + br - 1) >> p.br_log2;  // box pieces holding visible keys
            int phys = -1;
            uint32_t bytes = 0;
            const int tp = k0 + lane * br;  // first key of this lane's piece
            if (lane < npc) {
                phys = table[tp >> p.bs_log2];
                if (phys < 0 || phys >= p.num_blocks) {
                    set_error(p.error, PA_DEVERR_BLOCK_ID);
                    phys = -1;
                } else {
                    bytes = 2u * NDC * box_bytes;
                }
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
            unsigned char *kdst = stage_base + (size_t)stage * 2 * p.half_bytes;
            unsigned char *vdst = kdst + p.half_bytes;
            if (lane == 0) mbar_arrive_expect_tx(&full[stage], bytes);
            __syncwarp();
            if (phys >= 0) {
                const int32_t row = phys * p.bs + (tp & (p.bs - 1));
#pragma unroll
                for (int c2 = 0; c2 < NDC; ++c2) {
                    const size_t off = ((size_t)lane * NDC + c2) * box_bytes;
                    tma_load_3d(kdst + off, &p.tmap_k, c2 * 64, row, g, &full[stage], policy);
                    tma_load_3d(vdst + off, &p.tmap_v, c2 * 64, row, g, &full[stage], policy);
                }
            }
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
        }
        // every copy issued lands before the CTA retires
        volatile int never = 0;
        for (int st = 0; st < S; ++st)
            if (issued & (1u << st)) mbar_wait(&full[st], (issued_par >> st) & 1u, &never);
        mbar_wait(qbar, 0u, &never);
        return;
    }

    // ================= consumers: rows warp*16 .. warp*16+15 =================
    const int g4 = lane >> 2, t4 = lane & 3;
    const int rows = ntok * p.G;
    const int r_lo = warp * 16 + g4, r_hi = r_lo + 8;  // this lane's two rows
    const int qpos_lo = pos0 + r_lo / p.G, qpos_hi = pos0 + r_hi / p.G;
    const int warp_last_pos = pos0 + min(warp * 16 + 15, rows - 1) / p.G;  // furthest key any row sees
    const bool warp_live = warp * 16 < rows;

    if (!mbar_wait(qbar, 0u, abort_flag)) {
        *abort_flag = 1;
        if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
    }
    // Q as A fragments (m16 x k16 per k-step): row r at qs + r * D * E
    uint32_t qa[KS][4];
    {
        const unsigned char *r0 = qs + (size_t)r_lo * D * E, *r1 = qs + (size_t)r_hi * D * E;
        const bool v0 = r_lo < rows, v1 = r_hi < rows;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int c = ks * 16 + 2 * t4;
            qa[ks][0] = v0 ? *reinterpret_cast<const uint32_t *>(r0 + c * E) : 0u;
            qa[ks][1] = v1 ? *reinterpret_cast<const uint32_t *>(r1 + c * E) : 0u;
            qa[ks][2] = v0 ? *reinterpret_cast<const uint32_t *>(r0 + (c + 8) * E) : 0u;
            qa[ks][3] = v1 ? *reinterpret_cast<const uint32_t *>(r1 + (c + 8) * E) : 0u;
        }
    }
    float o[NO][4];
#pragma unroll
    for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

    // ldmatrix lane roles: K as B (non-transposed) and V as B (transposed)
    const int kb_key = (lane & 7) + ((lane >> 4) & 1) * 8, kb_col = ((lane >> 3) & 1);
    const int vb_key = (lane & 7) + ((lane >> 3) & 1) * 8, vb_col = (lane >> 4);

    int stage = 0;
    uint32_t phase = 0;
    for (int kt = 0; kt < ntiles; ++kt) {
        if (!*abort_flag && !mbar_wait(&full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            set_error(p.error, PA_DEVERR_TIMEOUT);
        }
        const int k0 = kt * p.KT;
        if (!*abort_flag && warp_live && k0 <= warp_last_pos) {
            unsigned char *kst = stage_base + (size_t)stage * 2 * p.half_bytes;
            unsigned char *vst = kst + p.half_bytes;
            const int nk16 = (min(p.KT, kend - k0) + 15) >> 4;  // 16-key groups with visible keys
            // V rows past the context end (unwritten pool slots in the last
            // block) get zero weight, but may hold anything: zero them before
            // they enter P V.  Every warp writes the same zeros before its own
            // reads, so no warp can see a stale row.
            const int vz0 = L - k0, vz1 = nk16 * 16;
            if (vz0 < vz1) {
                for (int i = lane; i < (vz1 - vz0) * (D / 8); i += 32)
                    *reinterpret_cast<uint4 *>(kv_chunk<D>(vst, vz0 + i / (D / 8), i % (D / 8), p.br_log2)) =
                        make_uint4(0u, 0u, 0u, 0u);
                fence_async_smem();  // ordered before the next tensor-map fill of this stage
                __syncwarp();
            }
            // One online-softmax step over NG groups of 16 keys (groups kg0 ..
            // kg0 + NG - 1, all loaded): S, mask, one max / rescale / sum, P V.
            auto step = [&](auto ng, int kg0) {
                constexpr int NG = decltype(ng)::value;
                // ---- S[16 rows x 16 NG keys] = Q K^T, one accumulation chain per 8 keys ----
                float sc[2 * NG][4];
#pragma unroll
                for (int nt = 0; nt < 2 * NG; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi) {
                        uint32_t bf[4];
                        ldmatrix_x4(bf, kv_chunk<D>(kst, (kg0 + gi) * 16 + kb_key, ks * 2 + kb_col, p.br_log2));
                        Op::mma(sc[2 * gi], qa[ks], bf[0], bf[1]);
                        Op::mma(sc[2 * gi + 1], qa[ks], bf[2], bf[3]);
                    }
                }
                // ---- causal mask, scores in the base-2 domain ----
                // sc[nt][0..1]: row lo, keys kc, kc+1 with kc = k0 + kg0*16 + nt*8 + 2*t4; [2..3]: row hi
                float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 2 * NG; ++nt) {
                    const int kc = k0 + kg0 * 16 + nt * 8 + 2 * t4;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        sc[nt][i] = kc + i <= qpos_lo ? sc[nt][i] * p.qscale : -INFINITY;
                        sc[nt][2 + i] = kc + i <= qpos_hi ? sc[nt][2 + i] * p.qscale : -INFINITY;
                        mx_lo = fmaxf(mx_lo, sc[nt][i]);
                        mx_hi = fmaxf(mx_hi, sc[nt][2 + i]);
                    }
                }
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
                const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
                // a row with no visible key yet keeps m = -inf: its weights are 0
                const float al_lo = mn_lo == -INFINITY ? 1.f : exp2_fast(m_lo - mn_lo);
                const float al_hi = mn_hi == -INFINITY ? 1.f : exp2_fast(m_hi - mn_hi);
                const float sub_lo = mn_lo == -INFINITY ? 0.f : mn_lo, sub_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
                float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2 * NG; ++nt) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        sc[nt][i] = exp2_fast(sc[nt][i] - sub_lo);  // masked: 2^-inf = 0
                        sc[nt][2 + i] = exp2_fast(sc[nt][2 + i] - sub_hi);
                        sum_lo += sc[nt][i];
                        sum_hi += sc[nt][2 + i];
                    }
                }
                sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 1);
                sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 2);
                sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 1);
                sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 2);
                l_lo = l_lo * al_lo + sum_lo;
                l_hi = l_hi * al_hi + sum_hi;
                m_lo = mn_lo;
                m_hi = mn_hi;
                if (al_lo != 1.f || al_hi != 1.f) {
#pragma unroll
                    for (int j = 0; j < NO; ++j) {
                        o[j][0] *= al_lo;
                        o[j][1] *= al_lo;
                        o[j][2] *= al_hi;
                        o[j][3] *= al_hi;
                    }
                }
                // ---- O[16 rows x D] += P V, one 16-key group at a time ----
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    // P as the A operand (m16 x k16), high and low 16-bit parts
                    const float *c0 = sc[2 * gi], *c1 = sc[2 * gi + 1];
                    uint32_t ph[4], pl[4];
                    ph[0] = Op::pack_p(c0[0], c0[1]);  // row lo, keys +2*t4
                    ph[1] = Op::pack_p(c0[2], c0[3]);  // row hi
                    ph[2] = Op::pack_p(c1[0], c1[1]);  // row lo, keys +8+2*t4
                    ph[3] = Op::pack_p(c1[2], c1[3]);  // row hi
                    {
                        const float2 h0 = Op::unpack(ph[0]), h1 = Op::unpack(ph[1]);
                        const float2 h2 = Op::unpack(ph[2]), h3 = Op::unpack(ph[3]);
                        pl[0] = Op::pack_p(c0[0] - h0.x, c0[1] - h0.y);
                        pl[1] = Op::pack_p(c0[2] - h1.x, c0[3] - h1.y);
                        pl[2] = Op::pack_p(c1[0] - h2.x, c1[1] - h2.y);
                        pl[3] = Op::pack_p(c1[2] - h3.x, c1[3] - h3.y);
                    }
                    const int vkey = (kg0 + gi) * 16 + vb_key;
#pragma unroll
                    for (int j2 = 0; j2 < NO / 2; ++j2) {
                        uint32_t vf[4];
                        ldmatrix_x4_trans(vf, kv_chunk<D>(vst, vkey, j2 * 2 + vb_col, p.br_log2));
                        Op::mma(o[2 * j2], ph, vf[0], vf[1]);
                        Op::mma(o[2 * j2 + 1], ph, vf[2], vf[3]);
                        Op::mma(o[2 * j2], pl, vf[0], vf[1]);
                        Op::mma(o[2 * j2 + 1], pl, vf[2], vf[3]);
                    }
                }
            };
            int kg = 0;
            for (; kg + 1 < nk16; kg += 2) step(std::integral_constant<int, 2>{}, kg);
            if (kg < nk16) step(std::integral_constant<int, 1>{}, kg);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == S) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (*abort_flag || !warp_live) return;
    // ---- normalise and store the rows of real tokens ----
    unsigned char *outb = static_cast<unsigned char *>(p.out);
    const float inv_lo = 1.f / l_lo, inv_hi = 1.f / l_hi;
    const size_t orow_lo = ((size_t)(q0 + t0 + r_lo / p.G) * p.Hq + (size_t)g * p.G + r_lo % p.G) * D;
    const size_t orow_hi = ((size_t)(q0 + t0 + r_hi / p.G) * p.Hq + (size_t)g * p.G + r_hi % p.G) * D;
#pragma unroll
    for (int j = 0; j < NO; ++j) {
        const int d = j * 8 + 2 * t4;
        if (r_lo < rows)
            *reinterpret_cast<uint32_t *>(outb + (orow_lo + d) * E) = Op::pack(o[j][0] * inv_lo, o[j][1] * inv_lo);
        if (r_hi < rows)
            *reinterpret_cast<uint32_t *>(outb + (orow_hi + d) * E) = Op::pack(o[j][2] * inv_hi, o[j][3] * inv_hi);
    }
}

}  // namespace pa
