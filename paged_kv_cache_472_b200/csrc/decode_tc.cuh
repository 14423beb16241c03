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
//   O^T[D x G] += V^T[D x 128] . P^T[128 x G]                    (M = D, N = G:
//       V^T is the staged V tile read MN-major; P^T is written by the softmax
//       threads, one token row each, over the K half of the same stage, which
//       the S product no longer needs; the weights enter as a high and a low
//       16-bit part, as in the other engines)
//
// Roles (warps 0-7 are the consumer warps of the kernel):
//   warps 0-3  softmax, one tensor-memory lane quarter each (32 tokens of S,
//              32 rows d of O); the epilogue (row sums, normalise, store)
//   warp 4     allocates tensor memory; lane 0 issues every tcgen05.mma, up
//              to two tiles of S ahead of the softmax; the whole warp patches
//              the fused step's new token into the staged tile and stores it
//   warps 5-7  follow the piece list (their arrivals keep the protocol
//              counts) and take part in the merge
// The running maximum of a head moves only when a tile's maximum exceeds it by
// more than 2^8 (weights stay below 256, exact in fp32 and safe in 16 bits);
// O^T in tensor memory is then rescaled, which is rare.  Every wait is
// bounded; on a timeout the CTA records PA_DEVERR_TIMEOUT, lets every issued
// product complete and frees its tensor memory before it leaves.
#pragma once

namespace pa {

constexpr int kTcSoftmaxWarps = 4;
constexpr int kTcMmaWarp = 4;
constexpr int kTcSBufs = 2;            // S buffers in tensor memory
constexpr int kTcTile = 128;           // tokens per tile: M of the S product
constexpr float kTcRescaleLog2 = 8.f;
constexpr int kTcBars = 10;            // sfull[2], pfull[2], odone[2], xchg[2], tdone, tfin

template <typename T, int G_>
struct TcEngine {
    static constexpr bool kTcgen05 = true;
    static constexpr int G = G_;
    static constexpr int kHeadsPerLane = G >= 32 ? G / 32 : 1;
    static constexpr int kTmemCols = 3 * G <= 64 ? 64 : (3 * G <= 128 ? 128 : 256);
    static constexpr int kColO = kTcSBufs * G;  // O^T after the S buffers
    static constexpr int kPRow = 2 * G;          // bytes of one token's P^T row (one 16-bit part)
    static_assert(G == 16 || G == 32 || G == 64, "group");
    // head held in slot k of `lane` after a reduce-scatter over the warp
    static __device__ __forceinline__ int own_head(int lane, int k) {
        return G == 16 ? (lane >> 1) : (G == 32 ? lane : 2 * lane + k);
    }
    // lane and slot holding head h after a reduce-scatter
    static __device__ __forceinline__ int src_lane(int h) { return G == 16 ? 2 * h : (G == 32 ? h : h >> 1); }
    static constexpr int src_slot(int h) { return G == 64 ? (h & 1) : 0; }
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

// G consecutive fp32 tensor-memory columns of this thread's lane.
template <int G>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float *v) {
    if constexpr (G == 16) {
        float (&w)[16] = *reinterpret_cast<float(*)[16]>(v);
        tmem_ld16(taddr, w);
    } else {
#pragma unroll
        for (int c = 0; c < G / 32; ++c) tmem_ld32(taddr + 32 * c, v + 32 * c);
    }
}

template <int G>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float *v) {
    if constexpr (G == 16) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(v[i]);
        tmem_st16u(taddr, w);
    } else {
#pragma unroll
        for (int c = 0; c < G / 32; ++c) tmem_st32(taddr + 32 * c, v + 32 * c);
    }
}

// Shared-memory layout of the staged tile in this engine (both halves):
// [d-chunk of 64][token row][128 B], the 16-byte chunks of a row swizzled by
// (row & 7).  P^T (one 16-bit part) over the K half: [token row][2G bytes],
// the 16-byte chunks swizzled by the 2G-byte pattern.
template <int G>
__device__ __forceinline__ uint32_t tc_p_chunk(int tok, int c) {
    constexpr int kRow = 2 * G;
    const int swz = kRow == 128 ? (tok & 7) : (kRow == 64 ? ((tok >> 1) & 3) : ((tok >> 2) & 1));
    return (uint32_t)(tok * kRow + ((c ^ swz) << 4));
}

template <typename T, int D, class Engine>
__device__ __forceinline__ void run_tc_consumers(const DecodeParams &p, DecodeCtl &ctl, const int *lens_s,
                                                 uint64_t *full, uint64_t *empty, uint64_t *qfull,
                                                 uint64_t *qempty, uint64_t *pdone, uint64_t *adone,
                                                 uint64_t *cbar, uint64_t *tcb, unsigned char *qarea,
                                                 unsigned char *stage_base, float *scratch,
                                                 volatile int *abort_flag, int tid, int warp, int lane) {
    using Op = Mma16<T>;
    constexpr int G = Engine::G;
    constexpr int E = 2;
    constexpr int NHL = Engine::kHeadsPerLane;
    constexpr int ST = kTcTile;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescQK = umma_idesc(ST, G, false, false, kBf16);
    constexpr uint32_t kIdescPV = umma_idesc(D, G, true, true, kBf16);
    constexpr uint32_t kChunk = (uint32_t)ST * 128u;  // one 64-wide d-chunk of a staged half
    static_assert(D == 128, "one O^T row per tensor-memory lane");
    uint64_t *sfull = tcb, *pfull = tcb + 2, *odone = tcb + 4, *xchg = tcb + 6, *tdone = tcb + 8, *tfin = tcb + 9;
    // scratch: red[2][4][G] (cross-warp exchange), mb[4][G] (running max per head,
    // one copy per warp), al[4][G] (rescale factors, one copy per warp)
    float *red = scratch;
    float *mb_w = scratch + 2 * 4 * G + warp * G;
    float *al_w = scratch + 3 * 4 * G + warp * G;
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
    // softmax warps: exchange counter and P V completions confirmed per barrier
    // every lane of the warp takes the same outcome, even at the time limit
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag) ? 1 : 0) != 0;
    };
    int xc = 0;
    int od_next[2] = {0, 0};
    auto od_wait = [&](int i) {
        int &nx = od_next[i & 1];
        for (; nx <= (i >> 1); ++nx)
            if (!wwait(&odone[i & 1], (uint32_t)nx & 1u)) return false;
        tc_fence_after();
        return true;
    };
    auto give_up = [&]() {
        *abort_flag = 1;
        set_error(p.error, PA_DEVERR_TIMEOUT);
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
            if (lane == 0) mbar_arrive(&qempty[qslot]);  // the MMA warp arrives by commit, after its last S product
        }
        qslot ^= 1;
        if (qslot == 0) qphase ^= 1u;
        const int ntiles = s.t_end - s.t_begin;

        if (warp == kTcMmaWarp) {
            // ================= tensor-core issue =================
            NewToken<D, E> nt;
            if (s.append_slot >= 0) nt.load(p, s.b, s.hg, lane);
            const int patch_tile = s.patch >= 0 ? (s.patch >> p.st_log2) - s.t_begin : -1;
            const int patch_tok = s.patch >= 0 ? s.patch - (s.patch >> p.st_log2) * ST : 0;
            const uint32_t q_addr = smem_u32(qarea + (size_t)my_qslot * p.q_bytes);
            int qk_n = 0;
            bool ok = !*abort_flag;
            auto issue_qk = [&](int i) {
                const int j = jt + i;
                if (ok && !wwait(&full[qk_stage], qk_phase)) ok = false;
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
            };
            for (int i = 0; i < ntiles; ++i) {
                while (qk_n < ntiles && qk_n < i + kTcSBufs) issue_qk(qk_n++);
                const int j = jt + i;
                if (lane == 0 && ok) {
                    if (!mbar_wait(&pfull[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag)) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        const int t = s.t_begin + i;
                        const int ntok = min(ST, s.L - t * ST);
                        const int n16 = (ntok + 15) >> 4;
                        unsigned char *kst = stage_base + (size_t)pv_stage * 2 * p.half_bytes;
                        const uint32_t pb = smem_u32(kst), vb = smem_u32(kst + p.half_bytes);
                        for (int kk = 0; kk < n16; ++kk) {
                            const uint64_t ad = umma_desc_sw128(vb + kk * 2048, kChunk, 1024);
                            const uint64_t bh = umma_desc_sw(pb + kk * 16 * Engine::kPRow, 8 * Engine::kPRow,
                                                             8 * Engine::kPRow, Engine::kPRow);
                            const uint64_t bl = umma_desc_sw(pb + ST * Engine::kPRow + kk * 16 * Engine::kPRow,
                                                             8 * Engine::kPRow, 8 * Engine::kPRow, Engine::kPRow);
                            umma_f16(tmem + Engine::kColO, ad, bh, kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                            umma_f16(tmem + Engine::kColO, ad, bl, kIdescPV, 1u);
                        }
                        umma_commit(&odone[j & 1]);
                        umma_commit(&empty[pv_stage]);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (++pv_stage == S) pv_stage = 0;
            }
            if (!ok) {
                if (lane == 0) give_up();
            } else if (s.append_slot >= 0) {
                nt.store(p, s.append_slot, s.hg, lane);  // the append proper
            }
        } else if (warp < kTcSoftmaxWarps) {
            // ================= softmax: one token (and one row d of O^T) per thread =================
            const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
            const int tok = warp * 32 + lane;
            const float qs = p.qscale;
            float lpart[G];
#pragma unroll
            for (int h = 0; h < G; ++h) lpart[h] = 0.f;
            float m_own[NHL];
#pragma unroll
            for (int k = 0; k < NHL; ++k) m_own[k] = -INFINITY;
            bool ok = !*abort_flag;
            int stage = (jt % S);  // the ring position of this piece's first tile
            for (int i = 0; i < ntiles && ok; ++i) {
                const int j = jt + i;
                const int t = s.t_begin + i;
                const int ntok = min(ST, s.L - t * ST);
                if (!wwait(&sfull[j % kTcSBufs], (uint32_t)(j / kTcSBufs) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float x[G];
                tmem_ld_cols<G>(tl + (uint32_t)(j % kTcSBufs) * G, x);
                const bool valid = tok < ntok;
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? x[h] * qs : -INFINITY;
                // ---- the tile's maximum per head over all 128 tokens ----
                {
                    float v[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) v[h] = x[h];
                    TcReduce<G, 16, true>::run(v, lane);
                    float *rb = red + (xc & 1) * 4 * G;
                    if (G != 16 || (lane & 1) == 0) {
#pragma unroll
                        for (int k = 0; k < NHL; ++k) rb[warp * G + Engine::own_head(lane, k)] = v[k];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xchg[xc & 1]);
                    if (!wwait(&xchg[xc & 1], (uint32_t)(xc >> 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    bool move = false;
                    float alpha[NHL];
#pragma unroll
                    for (int k = 0; k < NHL; ++k) {
                        const int h = Engine::own_head(lane, k);
                        const float mt = fmaxf(fmaxf(rb[h], rb[G + h]), fmaxf(rb[2 * G + h], rb[3 * G + h]));
                        alpha[k] = 1.f;
                        if (mt > m_own[k] + kTcRescaleLog2) {
                            alpha[k] = exp2_fast(m_own[k] - mt);  // 0 on the first tile
                            m_own[k] = mt;
                            move = true;
                        }
                    }
                    ++xc;
                    if (__any_sync(0xffffffffu, move)) {
                        // every warp takes the same decision from the same exchanged maxima
                        if (G != 16 || (lane & 1) == 0) {
#pragma unroll
                            for (int k = 0; k < NHL; ++k) {
                                mb_w[Engine::own_head(lane, k)] = m_own[k];
                                al_w[Engine::own_head(lane, k)] = alpha[k];
                            }
                        }
                        __syncwarp();
#pragma unroll
                        for (int h = 0; h < G; ++h) lpart[h] *= al_w[h];
                        if (i > 0) {
                            // O^T holds this piece's earlier tiles: rescale its columns,
                            // after P_{j-1} V_{j-1} has landed in it
                            if (!od_wait(j - 1)) {
                                ok = false;
                                break;
                            }
                            float o[G];
                            tmem_ld_cols<G>(tl + Engine::kColO, o);
#pragma unroll
                            for (int h = 0; h < G; ++h) o[h] *= al_w[h];
                            tmem_st_cols<G>(tl + Engine::kColO, o);
                            tmem_wait_st();
                        }
                    }
                }
                // ---- weights, row sums and P^T (two 16-bit parts) over the K half ----
                unsigned char *kst = stage_base + (size_t)stage * 2 * p.half_bytes;
                {
                    uint32_t hi[G / 2], lo[G / 2];
#pragma unroll
                    for (int h2 = 0; h2 < G / 2; ++h2) {
                        const float2 mm = *reinterpret_cast<const float2 *>(mb_w + 2 * h2);
                        const float e0 = exp2_fast(x[2 * h2] - mm.x), e1 = exp2_fast(x[2 * h2 + 1] - mm.y);
                        lpart[2 * h2] += e0;
                        lpart[2 * h2 + 1] += e1;
                        Op::split_p(e0, e1, hi[h2], lo[h2]);
                    }
#pragma unroll
                    for (int c = 0; c < G / 8; ++c) {
                        *reinterpret_cast<uint4 *>(kst + tc_p_chunk<G>(tok, c)) =
                            make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                        *reinterpret_cast<uint4 *>(kst + ST * Engine::kPRow + tc_p_chunk<G>(tok, c)) =
                            make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                    }
                }
                // V rows past the context inside the last 16-token group may hold
                // anything (unwritten pool rows or stale shared memory): zero them,
                // since a weight of 0 times a NaN is still NaN
                if (!valid && tok < ((ntok + 15) & ~15)) {
                    unsigned char *vst = kst + p.half_bytes;
#pragma unroll
                    for (int c2 = 0; c2 < D / 64; ++c2)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(vst + c2 * kChunk + tok * 128 + c * 16) = make_uint4(0, 0, 0, 0);
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
                float v[G];
#pragma unroll
                for (int h = 0; h < G; ++h) v[h] = lpart[h];
                TcReduce<G, 16, false>::run(v, lane);
                float *rb = red + (xc & 1) * 4 * G;
                if (G != 16 || (lane & 1) == 0) {
#pragma unroll
                    for (int k = 0; k < NHL; ++k) rb[warp * G + Engine::own_head(lane, k)] = v[k];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&xchg[xc & 1]);
                ok = wwait(&xchg[xc & 1], (uint32_t)(xc >> 1) & 1u);
                ++xc;
                if (ok) {
                    float l_own[NHL];
#pragma unroll
                    for (int k = 0; k < NHL; ++k) {
                        const int h = Engine::own_head(lane, k);
                        l_own[k] = (rb[h] + rb[G + h]) + (rb[2 * G + h] + rb[3 * G + h]);
                    }
                    float o[G];
                    tmem_ld_cols<G>(tl + Engine::kColO, o);
                    const int d = warp * 32 + lane;
                    if (s.nparts == 1) {
                        // every lane needs 1/l of every head: through this warp's copy area
                        if (G != 16 || (lane & 1) == 0) {
#pragma unroll
                            for (int k = 0; k < NHL; ++k) al_w[Engine::own_head(lane, k)] = 1.f / l_own[k];
                        }
                        __syncwarp();
                        unsigned char *outb = reinterpret_cast<unsigned char *>(p.out) +
                                              ((size_t)s.b * p.Hq + (size_t)s.hg * p.NHvr) * D * E;
#pragma unroll
                        for (int h = 0; h < G; ++h) Elem<T>::store1(outb + ((size_t)h * D + d) * E, o[h] * al_w[h]);
                    } else if (s.slot < p.max_slots) {
                        float *slot = p.partials + s.slot * p.slot_floats;
#pragma unroll
                        for (int h = 0; h < G; ++h) slot[h * D + d] = o[h];
                        if (warp == 0 && (G != 16 || (lane & 1) == 0)) {
#pragma unroll
                            for (int k = 0; k < NHL; ++k) {
                                const int h = Engine::own_head(lane, k);
                                slot[p.NHvr * D + h] = m_own[k];
                                slot[p.NHvr * D + p.NHvr + h] = l_own[k];
                            }
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
        if (s.nparts == 1) continue;
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
    flush_pending<T, D>(p, ctl, npend, adone, adone_par, abort_flag, cb, false, tid);

    // tensor memory: every product done and every reader past it before it is freed
    volatile int never = 0;
    if (warp < kTcSoftmaxWarps) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tdone);
    } else if (warp == kTcMmaWarp) {
        if (issued_any) {
            if (lane == 0) {
                umma_commit(tfin);
                mbar_wait(tfin, 0u, &never);
            }
        }
        __syncwarp();
        mbar_wait(tdone, 0u, &never);
        tc_fence_after();
        tmem_dealloc(tmem, Engine::kTmemCols);
    }
}

}  // namespace pa
