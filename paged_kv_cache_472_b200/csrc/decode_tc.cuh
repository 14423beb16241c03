// Consumer side of the decode kernel for large query-head groups (G = Hq/Hkv
// of 16, 32 or 64, D = 128, bf16 / fp16) on the 5th-generation tensor cores.
//
// The producer warp, the cut of the work, the partial slots and the
// log-sum-exp merge are those of paged_decode_kernel; only what happens to a
// staged tile differs.  A vr here is one request and one KV head, so every
// tile of 128 tokens is shared by the G query heads of that KV head:
//
//   S^T[128 tokens x G heads] = K_tile[128 x D] . Q^T[D x G]      (tcgen05.mma,
//       M = 128 tokens, N = G, both operands K-major from shared memory: the K
//       tile as the tensor-map boxes land it, Q as its own tensor-map box)
//   online softmax per head (fp32, base 2) over the tokens of the tile: the
//       tokens are the tensor-memory lanes, so a head's maximum is reduced
//       across the lanes of a warp (shuffles) and across the four warps (a
//       small shared-memory exchange on an mbarrier)
//   [O_hi^T | O_lo^T][D x 2G] += V^T[D x 128] . [P_hi^T | P_lo^T][128 x 2G]
//       (M = D, N = 2G: V^T is the staged V tile read MN-major; the weights
//       enter as a high and a low 16-bit part, as in the other engines, placed
//       side by side along N so that one product takes both; P^T is written by
//       the softmax threads, one token row each, over the K half of the same
//       stage, which the S product no longer needs; O^T = O_hi^T + O_lo^T at
//       the end)
//
// Roles (the CTA has 11 warps with this engine):
//   warps 0-7  softmax: warp w reads tensor-memory lane quarter w & 3 (32
//              tokens of S, 32 rows d of O^T) for half w >> 2 of the query
//              heads; the epilogue (row sums, normalise, store); the merge
//   warp 8     the producer (TMA boxes of K and V, q), as for every engine
//   warp 9     counts the arrivals of split pieces, as for every engine
//   warp 10    allocates tensor memory; lane 0 issues the S products (the next
//              tile's as soon as its K has landed and an S buffer is free);
//              the whole warp patches the fused step's new token into the
//              staged tile and stores it
//   warp 11    lane 0 issues the P V products, each as soon as P is written,
//              so that neither chain of products waits behind the other
// The running maximum of a head moves only when a tile's maximum exceeds it by
// more than 2^8 (weights stay below 256, exact in fp32 and safe in 16 bits);
// O^T in tensor memory is then rescaled, which is rare.  Every wait is
// bounded; on a timeout the CTA records PA_DEVERR_TIMEOUT, lets every issued
// product complete and frees its tensor memory before it leaves.
#pragma once

namespace pa {

constexpr int kTcSoftmaxWarps = kConsumerWarps;     // two per tensor-memory lane quarter
constexpr int kTcMmaWarp = kConsumerWarps + 2;      // S products (after the producer and the arrival warp)
constexpr int kTcPvWarp = kConsumerWarps + 3;       // P V products
constexpr int kTcThreads = (kConsumerWarps + 4) * 32;
constexpr int kTcSBufs = 2;            // S buffers in tensor memory
constexpr int kTcTile = 128;           // tokens per tile: M of the S product
constexpr float kTcRescaleLog2 = 8.f;
constexpr int kTcBars = 12;            // sfull[2], pfull[2], odone[2], xchg[2][2], tdone, tfin

template <typename T, int G_>
struct TcEngine {
    static constexpr bool kTcgen05 = true;
    static constexpr int kThreads = kTcThreads;
    static constexpr int G = G_;
    static constexpr int GH = G / 2;             // heads of one softmax thread (its half of the group)
    static constexpr int kTmemCols = 4 * G;     // two S buffers, then [O_hi^T | O_lo^T]
    static constexpr int kColO = kTcSBufs * G;  // O_hi^T after the S buffers, O_lo^T G columns on
    // [P_hi^T | P_lo^T]: 2G 16-bit values per token, in swizzle atoms of kPRow
    // bytes per token row (128-byte swizzle when the row is 128 bytes or more)
    static constexpr int kPRow = 4 * G < 128 ? 4 * G : 128;
    static constexpr int kPAtoms = 4 * G / kPRow;
    static constexpr int kShift = GH == 8 ? 2 : (GH == 16 ? 1 : 0);
    static_assert(G == 16 || G == 32 || G == 64, "group");
    // head (within the half) a lane holds after a reduce-scatter of GH values
    // over the warp; the lane writing it is the first of the 32 / GH that do
    static __device__ __forceinline__ int own_head(int lane) { return lane >> kShift; }
    static __device__ __forceinline__ bool head_writer(int lane) { return (lane & ((1 << kShift) - 1)) == 0; }
};

// Reduce-scatter of N per-lane values over the 32 lanes of a warp (maximum or
// sum).  Every step halves the values a lane keeps: the lane with bit O set
// keeps the upper half and sends the lower one.  Afterwards v[0 .. N/32)
// (one value when N < 32) holds the reduction over all lanes of the indices
// TcEngine::own_head names.
template <int N, int O, bool MAX>
struct TcReduce {
    static __device__ __forceinline__ void run(float *v, int lane) {
        if constexpr (O >= 1) {
            if constexpr (N > 1) {
                constexpr int H = N / 2;
                const bool up = (lane & O) != 0;
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const float keep = up ? v[i + H] : v[i];
                    const float send = up ? v[i] : v[i + H];
                    const float got = __shfl_xor_sync(0xffffffffu, send, O);
                    v[i] = MAX ? fmaxf(keep, got) : keep + got;
                }
                TcReduce<H, O / 2, MAX>::run(v, lane);
            } else {
                const float got = __shfl_xor_sync(0xffffffffu, v[0], O);
                v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
                TcReduce<1, O / 2, MAX>::run(v, lane);
            }
        }
    }
};

// N (8, 16 or a multiple of 32) consecutive fp32 tensor-memory columns of
// this thread's lane, waited for in the same statement.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float *v) {
    static_assert(N == 8 || N == 16 || N % 32 == 0, "columns");
    if constexpr (N == 8) {
        tmem_ld8(taddr, v);
    } else if constexpr (N == 16) {
        float (&w)[16] = *reinterpret_cast<float(*)[16]>(v);
        tmem_ld16(taddr, w);
    } else {
#pragma unroll
        for (int c = 0; c < N / 32; ++c) tmem_ld32(taddr + 32 * c, v + 32 * c);
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float *v) {
    static_assert(N == 8 || N == 16 || N % 32 == 0, "columns");
    if constexpr (N == 8) {
        tmem_st8(taddr, v);
    } else if constexpr (N == 16) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(v[i]);
        tmem_st16u(taddr, w);
    } else {
#pragma unroll
        for (int c = 0; c < N / 32; ++c) tmem_st32(taddr + 32 * c, v + 32 * c);
    }
}

// Shared-memory layout of the staged tile in this engine (both halves):
// [d-chunk of 64][token row][128 B], the 16-byte chunks of a row swizzled by
// (row & 7).  [P_hi^T | P_lo^T] over the K half, MN-major: [atom][token
// row][kPRow bytes], atom a holding N indices 64a .. 64a+63 (high parts at N
// = h, low parts at N = G + h), the 16-byte chunks swizzled by the kPRow-byte
// pattern.  Byte offset of the 16-byte chunk holding N indices n .. n+7 (n a
// multiple of 8) of token `tok`:
template <class Engine>
__device__ __forceinline__ uint32_t tc_p_chunk(int tok, int n) {
    constexpr int kRow = Engine::kPRow;
    const int swz = kRow == 128 ? (tok & 7) : (kRow == 64 ? ((tok >> 1) & 3) : ((tok >> 2) & 1));
    const int atom = n / (kRow / 2), c = (n % (kRow / 2)) / 8;
    return (uint32_t)(atom * kTcTile * kRow + tok * kRow + ((c ^ swz) << 4));
}

template <typename T, int D, class Engine>
__device__ __forceinline__ void run_tc_consumers(const DecodeParams &p, DecodeCtl &ctl, const int *lens_s,
                                                 uint64_t *full, uint64_t *empty, uint64_t *qfull,
                                                 uint64_t *qempty, uint64_t *pdone, uint64_t *adone,
                                                 uint64_t *cbar, uint64_t *mbar, uint64_t *tcb, unsigned char *qarea,
                                                 unsigned char *stage_base, float *scratch,
                                                 volatile int *abort_flag, int tid, int warp, int lane) {
    using Op = Mma16<T>;
    constexpr int G = Engine::G;
    constexpr int GH = Engine::GH;
    constexpr int E = 2;
    constexpr int ST = kTcTile;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescQK = umma_idesc(ST, G, false, false, kBf16);
    constexpr uint32_t kIdescPV = umma_idesc(D, 2 * G, true, true, kBf16);
    constexpr uint32_t kChunk = (uint32_t)ST * 128u;  // one 64-wide d-chunk of a staged half
    static_assert(D == 128, "one O^T row per tensor-memory lane");
    uint64_t *sfull = tcb, *pfull = tcb + 2, *odone = tcb + 4, *tdone = tcb + 10, *tfin = tcb + 11;
    const int quad = warp & 3, half = (warp >> 2) & 1;  // softmax warps: lane quarter, head half
    uint64_t *xchg = tcb + 6 + 2 * half;                  // this half's four warps
    // scratch: red[2 halves][2 buffers][4 quarters][GH] (exchange), mb[8 warps][GH]
    // (running maximum per head, one copy per warp), al[8][GH] (rescale factors)
    float *red = scratch + half * 8 * GH;
    float *mb_w = scratch + 16 * GH + (warp & 7) * GH;
    float *al_w = scratch + 24 * GH + (warp & 7) * GH;
    const uint32_t tmem = ctl.tmem_base;
    const int S = p.stages;

    ConsumerBarrier cb{cbar, 0u};
    int qslot = 0;
    uint32_t qphase = 0;
    int npend = 0;
    uint32_t adone_par = 0;
    int jt = 0;          // tiles of this CTA before the current piece
    // MMA warp: K/V ring cursors (full waits for S products, empty commits for P V products)
    int qk_stage = 0, pv_stage = 0;
    uint32_t qk_phase = 0;
    bool issued_any = false;
    // every lane of the warp takes the same outcome, even at the time limit
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag) ? 1 : 0) != 0;
    };
    auto wspin = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort_flag) ? 1 : 0) != 0;
    };
    // softmax warps: exchange counter and P V completions confirmed per barrier
    int xc = 0;
    int od_next[2] = {0, 0};
    auto od_wait = [&](int i) {
        int &nx = od_next[i & 1];
        for (; nx <= (i >> 1); ++nx)
            if (!wspin(&odone[i & 1], (uint32_t)nx & 1u)) return false;
        tc_fence_after();
        return true;
    };
    auto give_up = [&]() {
        *abort_flag = 1;
        set_error(p.error, PA_DEVERR_TIMEOUT);
    };
    // the exchange of per-warp values (maxima or sums) of this half's heads
    // over the four lane quarters: returns the combination for own_head(lane)
    auto exchange = [&](float v, bool is_max, bool &ok) {
        float *rb = red + (xc & 1) * 4 * GH;
        if (Engine::head_writer(lane)) rb[quad * GH + Engine::own_head(lane)] = v;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xchg[xc & 1]);
        ok = wspin(&xchg[xc & 1], (uint32_t)(xc >> 1) & 1u);
        ++xc;
        const int h = Engine::own_head(lane);
        const float a = rb[h], b = rb[GH + h], c = rb[2 * GH + h], d = rb[3 * GH + h];
        return is_max ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
    };

    for (;;) {
        if (!wwait(&qfull[qslot], qphase)) {
            if (lane == 0) give_up();
            break;
        }
        const Seg s = ctl.segs[qslot];
        if (s.b < 0) break;
        const int my_qslot = qslot;
        if (warp != kTcMmaWarp) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[qslot]);  // the S warp arrives by commit, after its last S product
        }
        qslot ^= 1;
        if (qslot == 0) qphase ^= 1u;
        const int ntiles = s.t_end - s.t_begin;

        if (warp == kTcMmaWarp) {
            // ================= S products =================
            NewToken<D, E> nt;
            if (s.append_slot >= 0) nt.load(p, s.b, s.hg, lane);
            const int patch_tile = s.patch >= 0 ? (s.patch >> p.st_log2) - s.t_begin : -1;
            const int patch_tok = s.patch >= 0 ? s.patch - (s.patch >> p.st_log2) * ST : 0;
            const uint32_t q_addr = smem_u32(qarea + (size_t)my_qslot * p.q_bytes);
            bool ok = !*abort_flag;
            for (int i = 0; i < ntiles; ++i) {
                // S_i = K_i Q^T into buffer j % 2, free once P_{j-2} is written
                const int j = jt + i;
                if (ok && !wwait(&full[qk_stage], qk_phase)) ok = false;
                if (ok && j >= kTcSBufs && !wwait(&pfull[j & 1], (uint32_t)((j - kTcSBufs) >> 1) & 1u)) ok = false;
                if (ok) {
                    unsigned char *kst = stage_base + (size_t)qk_stage * 2 * p.half_bytes;
                    if (i == patch_tile) nt.patch(kst, kst + p.half_bytes, patch_tok, 0, p, lane);
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t kb = smem_u32(kst);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint64_t ad = umma_desc_sw128(kb + (ks >> 2) * kChunk + (ks & 3) * 32, 16, 1024);
                            const uint64_t bd =
                                umma_desc_sw128(q_addr + (ks >> 2) * (G * 128) + (ks & 3) * 32, 16, 1024);
                            umma_f16(tmem + (uint32_t)(j % kTcSBufs) * G, ad, bd, kIdescQK, ks > 0 ? 1u : 0u);
                        }
                        umma_commit(&sfull[j % kTcSBufs]);
                        if (i == ntiles - 1) umma_commit(&qempty[my_qslot]);  // Q is read for the last time
                    }
                    issued_any = true;
                }
                __syncwarp();
                if (++qk_stage == S) {
                    qk_stage = 0;
                    qk_phase ^= 1u;
                }
            }
            if (!ok) {
                if (lane == 0) give_up();
            } else if (s.append_slot >= 0) {
                nt.store(p, s.append_slot, s.hg, lane);  // the append proper
            }
            jt += ntiles;
            continue;  // the issuing warps take no part in the partials and the merge
        }
        if (warp == kTcPvWarp) {
            // ================= P V products =================
            bool ok = !*abort_flag;
            for (int i = 0; i < ntiles; ++i) {
                const int j = jt + i;
                if (ok && !wwait(&pfull[j & 1], (uint32_t)(j >> 1) & 1u)) ok = false;
                if (ok && lane == 0) {
                    tc_fence_after();
                    const int t = s.t_begin + i;
                    const int ntok = min(ST, s.L - t * ST);
                    const int n16 = (ntok + 15) >> 4;
                    unsigned char *kst = stage_base + (size_t)pv_stage * 2 * p.half_bytes;
                    const uint32_t pb = smem_u32(kst), vb = smem_u32(kst + p.half_bytes);
                    for (int kk = 0; kk < n16; ++kk) {
                        const uint64_t ad = umma_desc_sw128(vb + kk * 2048, kChunk, 1024);
                        const uint64_t bd = umma_desc_sw(pb + kk * 16 * Engine::kPRow, ST * Engine::kPRow,
                                                         8 * Engine::kPRow, Engine::kPRow);
                        umma_f16(tmem + Engine::kColO, ad, bd, kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&odone[j & 1]);
                    umma_commit(&empty[pv_stage]);
                }
                if (ok) issued_any = true;
                __syncwarp();
                if (++pv_stage == S) pv_stage = 0;
            }
            if (!ok && lane == 0) give_up();
            jt += ntiles;
            continue;
        }

        // ================= softmax: one token (and one row d of O^T) per thread, half the heads =================
        {
            const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
            const uint32_t col_s = (uint32_t)half * GH;            // this half's columns of S
            const uint32_t col_o = (uint32_t)Engine::kColO + half * GH;
            const int tok = quad * 32 + lane;
            const float qs = p.qscale;
            float lpart[GH];
#pragma unroll
            for (int h = 0; h < GH; ++h) lpart[h] = 0.f;
            float m_own = -INFINITY;  // running maximum of head own_head(lane) of this half
            bool ok = !*abort_flag;
            int stage = (jt % S);  // the ring position of this piece's first tile
            for (int i = 0; i < ntiles && ok; ++i) {
                const int j = jt + i;
                const int t = s.t_begin + i;
                const int ntok = min(ST, s.L - t * ST);
                if (!wspin(&sfull[j % kTcSBufs], (uint32_t)(j / kTcSBufs) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float x[GH];
                tmem_ld_cols<GH>(tl + (uint32_t)(j % kTcSBufs) * G + col_s, x);
                const bool valid = tok < ntok;
#pragma unroll
                for (int h = 0; h < GH; ++h) x[h] = valid ? x[h] * qs : -INFINITY;
                // ---- the tile's maximum per head over all 128 tokens ----
                {
                    float v[GH];
#pragma unroll
                    for (int h = 0; h < GH; ++h) v[h] = x[h];
                    TcReduce<GH, 16, true>::run(v, lane);
                    const float mt = exchange(v[0], true, ok);
                    if (!ok) break;
                    float alpha = 1.f;
                    bool move = false;
                    if (mt > m_own + kTcRescaleLog2) {
                        alpha = exp2_fast(m_own - mt);  // 0 on the first tile
                        m_own = mt;
                        move = true;
                    }
                    if (__any_sync(0xffffffffu, move)) {
                        // the four warps of this half take the same decision from the same maxima
                        if (Engine::head_writer(lane)) {
                            mb_w[Engine::own_head(lane)] = m_own;
                            al_w[Engine::own_head(lane)] = alpha;
                        }
                        __syncwarp();
#pragma unroll
                        for (int h = 0; h < GH; ++h) lpart[h] *= al_w[h];
                        if (i > 0) {
                            // O^T holds this piece's earlier tiles: rescale this half's
                            // columns once P_{j-1} V_{j-1} has landed in it
                            if (!od_wait(j - 1)) {
                                ok = false;
                                break;
                            }
                            float o[GH];
#pragma unroll
                            for (int part = 0; part < 2; ++part) {
                                tmem_ld_cols<GH>(tl + col_o + part * G, o);
#pragma unroll
                                for (int h = 0; h < GH; ++h) o[h] *= al_w[h];
                                tmem_st_cols<GH>(tl + col_o + part * G, o);
                            }
                            tmem_wait_st();
                        }
                    }
                }
                // ---- weights, row sums and P^T (two 16-bit parts) over the K half ----
                unsigned char *kst = stage_base + (size_t)stage * 2 * p.half_bytes;
                {
                    uint32_t hi[GH / 2], lo[GH / 2];
#pragma unroll
                    for (int h2 = 0; h2 < GH / 2; ++h2) {
                        const float2 mm = *reinterpret_cast<const float2 *>(mb_w + 2 * h2);
                        const float e0 = exp2_fast(x[2 * h2] - mm.x), e1 = exp2_fast(x[2 * h2 + 1] - mm.y);
                        lpart[2 * h2] += e0;
                        lpart[2 * h2 + 1] += e1;
                        Op::split_p(e0, e1, hi[h2], lo[h2]);
                    }
#pragma unroll
                    for (int c = 0; c < GH / 8; ++c) {
                        const int n = half * GH + 8 * c;  // this chunk's first head
                        *reinterpret_cast<uint4 *>(kst + tc_p_chunk<Engine>(tok, n)) =
                            make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                        *reinterpret_cast<uint4 *>(kst + tc_p_chunk<Engine>(tok, G + n)) =
                            make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                    }
                }
                // V rows past the context inside the last 16-token group may hold
                // anything (unwritten pool rows or stale shared memory): zero them,
                // since a weight of 0 times a NaN is still NaN (each half zeroes one d-chunk)
                if (!valid && tok < ((ntok + 15) & ~15)) {
                    unsigned char *vrow = kst + p.half_bytes + half * kChunk + tok * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
                }
                // confirm P_{j-2} V_{j-2} before P_j is published, so that no
                // barrier of the P V completions runs two phases ahead of us
                if (j >= 2 && !od_wait(j - 2)) {
                    ok = false;
                    break;
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[j & 1]);
                if (++stage == S) stage = 0;
            }
            // ---- epilogue: row sums over the tokens, O^T / l, store ----
            if (ok && ntiles > 0 && od_wait(jt + ntiles - 1)) {
                float v[GH];
#pragma unroll
                for (int h = 0; h < GH; ++h) v[h] = lpart[h];
                TcReduce<GH, 16, false>::run(v, lane);
                const float l_own = exchange(v[0], false, ok);
                if (ok) {
                    float o[GH], o_lo[GH];
                    tmem_ld_cols<GH>(tl + col_o, o);
                    tmem_ld_cols<GH>(tl + col_o + G, o_lo);
#pragma unroll
                    for (int h = 0; h < GH; ++h) o[h] += o_lo[h];
                    const int d = quad * 32 + lane;
                    const int h0 = half * GH;  // first head of this half within the vr
                    if (s.nparts == 1) {
                        // every lane needs 1/l of every head: through this warp's copy area
                        if (Engine::head_writer(lane)) al_w[Engine::own_head(lane)] = 1.f / l_own;
                        __syncwarp();
                        unsigned char *outb = reinterpret_cast<unsigned char *>(p.out) +
                                              ((size_t)s.b * p.Hq + (size_t)s.hg * p.NHvr + h0) * D * E;
#pragma unroll
                        for (int h = 0; h < GH; ++h) Elem<T>::store1(outb + ((size_t)h * D + d) * E, o[h] * al_w[h]);
                    } else if (s.slot < p.max_slots) {
                        float *slot = p.partials + s.slot * p.slot_floats;
#pragma unroll
                        for (int h = 0; h < GH; ++h) slot[(h0 + h) * D + d] = o[h];
                        if (quad == 0 && Engine::head_writer(lane)) {
                            const int h = h0 + Engine::own_head(lane);
                            slot[p.NHvr * D + h] = m_own;
                            slot[p.NHvr * D + p.NHvr + h] = l_own;
                        }
                    } else if (tid == 0) {
                        set_error(p.error, PA_DEVERR_WORKSPACE);
                    }
                    __syncwarp();
                }
            }
            if (!ok) {
                if (lane == 0) give_up();
            }
        }
        jt += ntiles;

        // partial piece: the arrival warp counts it once every consumer warp is past it
        // (the merge grid combines the pieces instead when split_merge is set)
        if (s.nparts == 1 || p.split_merge) continue;
        __syncwarp();
        if (tid == 0) ctl.pending[npend] = s;
        if (lane == 0) mbar_arrive(&pdone[npend]);
        if (++npend == kMaxPending) {
            flush_pending<T, D>(p, ctl, npend, adone, adone_par, abort_flag, cb, true, tid);
            adone_par ^= 1u;
            npend = 0;
        }
    }

    volatile int never = 0;
    if (warp == kTcMmaWarp || warp == kTcPvWarp) {
        // both issuers' products complete (tfin counts one arrival from each),
        // and every reader is past tensor memory, before it is freed
        if (lane == 0) {
            if (issued_any) umma_commit(tfin);
            else mbar_arrive(tfin);
        }
        if (warp == kTcPvWarp) return;
        if (lane == 0) mbar_wait(tfin, 0u, &never);
        __syncwarp();
        mbar_wait(tdone, 0u, &never);
        tc_fence_after();
        tmem_dealloc(tmem, Engine::kTmemCols);
        return;
    }
    // softmax warps: past their last tensor-memory read
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tdone);
    // close the list for the arrival warp, then merge what this CTA completed
    if (tid == 0) ctl.pending[npend].b = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&pdone[npend]);
    flush_pending<T, D>(p, ctl, npend, adone, adone_par, abort_flag, cb, false, tid, stage_base,
                        (uint32_t)S * 2u * p.half_bytes, mbar);
}

}  // namespace pa
