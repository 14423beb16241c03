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
// Its 128 rows are the QT tokens x G query heads of that KV head (row r =
// token r / G, head r % G), so every K/V tile staged in shared memory serves
// the whole head group.  The CTA streams keys 0 .. pos(last token) in tiles
// of 128 and masks, per row, the keys past the row's own position.  Tiles
// holding the latest tokens see the most keys; the grid runs them first.
//
// Inside a CTA (5th-generation tensor cores, accumulators in tensor memory):
//   warps 0,10 producers of K and of V: each walks the block table (one tile
//              ahead) and fills its own ring of slots with tensor-map boxes
//              ([d-block][key][128 B], 128-byte swizzle: the canonical K-major
//              layout for K, MN-major for V), so K never queues behind a V
//              slot that a product still holds;
//   warp 1     allocates tensor memory; one lane issues every tcgen05.mma:
//                S_j = Q K_j^T   (M 128 rows, N 128 keys, into one of three
//                                 S buffers, up to three tiles ahead of the
//                                 softmax),
//                O  += P_j V_j   (M 128 rows, N = D, K = keys; P read from
//                                 tensor memory, where the softmax wrote it
//                                 over S_j, in two 16-bit parts, high and
//                                 low, as in decode);
//   warps 2-9  softmax: two threads per row (tensor-memory lane = row), one
//              for each half of the key columns (and of the O columns).  They
//              copy the q rows into the swizzled Q tile, then per key tile
//              read their half of the S row, mask, exchange the row maximum
//              with the partner (a two-warp mbarrier), run the fp32 online
//              softmax in the base-2 domain, write P (high and low parts) into
//              the S buffer they read, and at the end combine the two row
//              sums, read O, divide and store the output row.
// The tensor pipe runs its products in issue order, so S_{j+3} (issued after
// P_j V_j) never overwrites P_j before it is read, and the softmax of tile j
// never waits for P_{j-1} V_{j-1}: only a rescale of O does.
// The running maximum is moved only when a tile's maximum exceeds it by more
// than 2^8 (weights stay below 256, exact in fp32 and safe in 16 bits); the
// rescale of O in tensor memory is then rare.  The final division uses the
// same maximum as every weight, so the result is the plain softmax.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace pa {

constexpr int kPrefillRows = 128;     // rows per CTA: M of every tensor-core product
constexpr int kPrefillKT = 128;       // keys per tile: N of S, K of P V
constexpr int kPrefillSoftmaxWarps = 8;
constexpr int kPrefillVWarp = 2 + kPrefillSoftmaxWarps;             // the V producer
constexpr int kPrefillThreads = (3 + kPrefillSoftmaxWarps) * 32;  // K producer, MMA, softmax, V producer
constexpr int kPrefillSBufs = 3;      // S / P buffers in tensor memory
constexpr int kPrefillTmemCols = 512; // S / P buffers (3 x 128 columns) + O (D columns), power of two
constexpr int kPrefillMaxSlots = 8;   // K / V ring slots
constexpr float kPrefillRescaleLog2 = 8.f;

struct PrefillParams {
    CUtensorMap tmap_k;  // box {64 d, br rows, 1 head} on [d, token row, head] views of the pools
    CUtensorMap tmap_v;
    const void *q;       // [T, Hq, D]
    void *out;           // [T, Hq, D]
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *query_start;
    int32_t *error;      // device error word or nullptr
    float qscale;        // |scale| * log2(e)
    uint32_t qflip;      // 0x80008000 when scale < 0: q enters negated, so scores keep their order
    int32_t B, Hq, Hkv, G, g_log2, bs, bs_log2, num_blocks, max_blocks;
    int32_t QT;          // new tokens per CTA (QT * G = kPrefillRows)
    int32_t br_log2;     // rows of one box = min(kPrefillKT, bs)
    int32_t nslots;      // ring slots, even: K of tile j in slot j mod (nslots/2), V of tile j in the second half
    int32_t num_qtiles;  // tiles of QT tokens the grid covers per request
    uint32_t off_ring, slot_bytes;  // shared-memory layout (from the 1024-aligned base; Q at 0)
};
static_assert(offsetof(PrefillParams, tmap_k) % 64 == 0 && offsetof(PrefillParams, tmap_v) % 64 == 0,
              "tensor maps must be 64-byte aligned");

template <typename T, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1) paged_prefill_kernel(const __grid_constant__ PrefillParams p) {
    using Op = Mma16<T>;
    constexpr int E = 2;
    constexpr int KT = kPrefillKT;
    constexpr int KS = D / 16;                         // k-steps of S over d
    constexpr int NDC = D / 64;                        // 64-wide d-blocks
    constexpr uint32_t kBlk = kPrefillRows * 128u;     // one 64-column block of a 128-row operand: 16 KB
    constexpr uint32_t kSlotBlk = KT * 128u;           // one d-block of a K / V slot
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescPV = umma_idesc(kPrefillRows, D, false, true, kBf16);
    constexpr uint32_t kColO = kPrefillSBufs * KT;     // tensor-memory column of O
    static_assert(kPrefillSBufs * KT + D <= kPrefillTmemCols, "tensor memory");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw;  // the plan leaves no room to realign: checked below
    // mbarriers: full[], empty[] (ring), sfull[3], pfull[2], odone[2], qfull, fin, xchg[4][2]
    constexpr int kOffSfull = 2 * kPrefillMaxSlots, kOffPfull = kOffSfull + kPrefillSBufs;
    constexpr int kOffOdone = kOffPfull + 2, kOffQfull = kOffOdone + 2, kOffFin = kOffQfull + 1;
    constexpr int kOffXchg = kOffFin + 1, kBars = kOffXchg + 8;
    __shared__ uint64_t bars[kBars];
    __shared__ float red_s[2][2][kPrefillRows];  // [tile parity][column half][row]: row max / row sum
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NH = p.nslots / 2;  // K slots 0 .. NH-1, V slots NH .. 2NH-1
    uint64_t *full = bars, *empty = bars + kPrefillMaxSlots;
    // sfull (one per S buffer), pfull and odone (one per tile parity): no
    // barrier's phase can run two ahead of a thread that waits on it by parity
    uint64_t *sfull = bars + kOffSfull, *pfull = bars + kOffPfull, *odone = bars + kOffOdone;
    uint64_t *qfull = bars + kOffQfull, *fin = bars + kOffFin;
    uint64_t *xchg = bars + kOffXchg;  // [lane quarter][parity]: the two softmax warps of the same rows
    volatile int *abort_flag = &abort_s;

    if (smem_u32(smem_raw) & 1023u) {  // the 128-byte swizzle needs 1024-byte aligned tiles
        if (tid == 0) set_error(p.error, PA_DEVERR_SMEM);
        return;
    }
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
    const int pos0 = L - n + t0;            // position of the tile's first token
    const int kend = pos0 + ntok;           // keys 0 .. kend-1 are visible to some row
    const int ntiles = (kend + KT - 1) / KT;
    const int nk_last = kend - (ntiles - 1) * KT;  // keys of the last tile holding visible keys
    const int n16_last = (nk_last + 15) >> 4;      // its 16-key groups

    if (tid == 0) {
        for (int s = 0; s < 2 * NH; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < kPrefillSBufs; ++i) mbar_init(&sfull[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pfull[i], kPrefillSoftmaxWarps);
            mbar_init(&odone[i], 1);
        }
        mbar_init(qfull, kPrefillSoftmaxWarps);
        mbar_init(fin, 1);
        for (int i = 0; i < 8; ++i) mbar_init(&xchg[i], 2);
        abort_s = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base_s, kPrefillTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    unsigned char *ring = smem + p.off_ring;

    if (warp == 0 || warp == kPrefillVWarp) {
        // ================= producers: K (warp 0) and V =================
        const int mat = warp == 0 ? 0 : 1;
        const CUtensorMap *map = mat ? &p.tmap_v : &p.tmap_k;
        const int base = mat * NH;  // this matrix's ring slots: base .. base + NH - 1
        const uint64_t policy = policy_evict_normal();  // K/V are read by every q-tile of the request
        const int32_t *table = p.block_tables + (size_t)b * p.max_blocks;
        const int br = 1 << p.br_log2;
        const uint32_t box_bytes = 128u << p.br_log2;
        // physical block of this lane's box piece of tile j (-1: no piece, or a bad entry)
        auto lookup = [&](int j) {
            const int k0 = j * KT;
            const int npc = (min(KT, kend - k0) + br - 1) >> p.br_log2;  // pieces holding visible keys
            int phys = -1;
            if (lane < npc) {
                phys = table[(k0 + lane * br) >> p.bs_log2];
                if (phys < 0 || phys >= p.num_blocks) {
                    set_error(p.error, PA_DEVERR_BLOCK_ID);
                    phys = -1;
                }
            }
            return phys;
        };
        uint32_t issued = 0, issued_par = 0;
        bool ok = true;
        int phys = lookup(0);
        for (int j = 0; j < ntiles; ++j) {
            const int cur = phys;
            if (j + 1 < ntiles) phys = lookup(j + 1);  // the next tile's entries load while this one waits
            uint32_t bytes = cur >= 0 ? NDC * box_bytes : 0u;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
            const int slot = base + j % NH;
            const uint32_t par = (uint32_t)(j / NH) & 1u;
            if (!mbar_wait(&empty[slot], par ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
            __syncwarp();
            if (cur >= 0) {
                const int32_t row = cur * p.bs + ((j * KT + lane * br) & (p.bs - 1));
                unsigned char *dst = ring + (size_t)slot * p.slot_bytes + (size_t)lane * box_bytes;
#pragma unroll
                for (int c = 0; c < NDC; ++c)
                    tma_load_3d(dst + c * kSlotBlk, map, c * 64, row, g, &full[slot], policy);
            }
            issued |= 1u << slot;
            issued_par = (issued_par & ~(1u << slot)) | (par << slot);
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
        }
        // every copy issued lands before the CTA retires
        volatile int never = 0;
        for (int st = base; st < base + NH; ++st)
            if (issued & (1u << st)) mbar_wait(&full[st], (issued_par >> st) & 1u, &never);
    } else if (warp == 1) {
        // ================= MMA issue (one lane) =================
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(smem), r_addr = smem_u32(ring);
            bool ok = mbar_wait(qfull, 0u, abort_flag);
            bool issued_any = false;
            // O += P_i V_i for tile i (P high part, then low part)
            auto pv = [&](int i) {
                if (!ok) return;
                const int sv = NH + i % NH;
                const uint32_t par = (uint32_t)(i / NH) & 1u;
                if (!mbar_wait(&pfull[i & 1], (uint32_t)(i >> 1) & 1u, abort_flag) ||
                    !mbar_wait(&full[sv], par, abort_flag)) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                const int n16 = i == ntiles - 1 ? n16_last : KT / 16;
                const uint32_t vb = r_addr + (uint32_t)sv * p.slot_bytes;
                // P_i in buffer i % 3: keys 16kk .. 16kk+15 in columns 16kk .. 16kk+7
                // (high parts) and 16kk+8 .. 16kk+15 (low parts), two keys per column
                const uint32_t pa = tmem + (uint32_t)(i % kPrefillSBufs) * KT;
                for (int kk = 0; kk < n16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(vb + kk * 2048, kSlotBlk, 1024);
                    umma_f16_ts(tmem + kColO, pa + kk * 16, bd, kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                    umma_f16_ts(tmem + kColO, pa + kk * 16 + 8, bd, kIdescPV, 1u);
                }
                umma_commit(&odone[i & 1]);
                umma_commit(&empty[sv]);
                issued_any = true;
            };
            // S_j = Q K_j^T into buffer j % 3, which held P_{j-3}: issued after P_{j-3} V_{j-3}
            auto s_issue = [&](int j) {
                if (!ok) return;
                const int sk = j % NH;
                const uint32_t par = (uint32_t)(j / NH) & 1u;
                if (!mbar_wait(&full[sk], par, abort_flag)) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                const int N = j == ntiles - 1 ? n16_last * 16 : KT;
                const uint32_t idesc = umma_idesc(kPrefillRows, N, false, false, kBf16);
                const uint32_t kb = r_addr + (uint32_t)sk * p.slot_bytes;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const uint64_t ad = umma_desc_sw128(q_addr + (ks >> 2) * kBlk + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(kb + (ks >> 2) * kSlotBlk + (ks & 3) * 32, 16, 1024);
                    umma_f16(tmem + (uint32_t)(j % kPrefillSBufs) * KT, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&sfull[j % kPrefillSBufs]);
                umma_commit(&empty[sk]);
                issued_any = true;
            };
            for (int j = 0; j < kPrefillSBufs && j < ntiles; ++j) s_issue(j);
            for (int i = 0; i < ntiles && ok; ++i) {
                pv(i);
                if (i + kPrefillSBufs < ntiles) s_issue(i + kPrefillSBufs);
            }
            if (!ok) {
                *abort_flag = 1;
                set_error(p.error, PA_DEVERR_TIMEOUT);
            }
            if (issued_any) {
                // every product issued completes before tensor memory is released
                umma_commit(fin);
                volatile int never = 0;
                mbar_wait(fin, 0u, &never);
            }
        }
    } else {
        // ================= softmax: two threads per row =================
        constexpr int HC = KT / 2;            // S columns per thread
        constexpr int HD = D / 2;             // O columns per thread
        const int half = (warp - 2) >> 2;     // column half
        const int quad = warp & 3;            // tensor-memory lane quarter of this warp
        const int row = quad * 32 + lane;
        const int sid = tid - 64;             // 0 .. 255 over the softmax warps
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);  // this warp's lanes
        uint64_t *xb = xchg + quad * 2;
        const int tok = row >> p.g_log2, hj = row & (p.G - 1);
        const bool valid = tok < ntok;
        const size_t grow = ((size_t)(q0 + t0 + tok) * p.Hq + (size_t)g * p.G + hj) * D;  // q / out row
        // ---- Q tile: half of row `row`, K-major with the 128-byte swizzle ----
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.q) + grow * E);
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                const int c = half * (D / 16) + i;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (valid) {
                    v = __ldg(src + c);
                    v.x ^= p.qflip;
                    v.y ^= p.qflip;
                    v.z ^= p.qflip;
                    v.w ^= p.qflip;
                }
                *reinterpret_cast<uint4 *>(smem + (c >> 3) * kBlk + row * 128 + (((c & 7) ^ (row & 7)) << 4)) = v;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        const int pos_row = pos0 + (valid ? tok : ntok - 1);  // rows past the tokens mirror the last token
        const float qs = p.qscale;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        // P V completions, confirmed per barrier in order: odone[i & 1] phase
        // i >> 1 is P_i V_i, and P_{i+2} V_{i+2} cannot complete before the
        // softmax of tile i+2 has run, so a parity wait never skips a phase
        int od_next[2] = {0, 0};
        auto od_wait = [&](int i) {
            int &nx = od_next[i & 1];
            for (; nx <= (i >> 1); ++nx)
                if (!mbar_wait(&odone[i & 1], (uint32_t)nx & 1u, abort_flag)) return false;
            tc_fence_after();
            return true;
        };
        for (int j = 0; j < ntiles; ++j) {
            const int k0 = j * KT;
            const uint32_t sb = tl + (uint32_t)(j % kPrefillSBufs) * KT;  // S_j, then P_j
            if (!mbar_wait(&sfull[j % kPrefillSBufs], (uint32_t)(j / kPrefillSBufs) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[HC];
            tmem_ld32(sb + half * HC, s);
            tmem_ld32(sb + half * HC + 32, s + 32);
            // keys past the row's position (or past the keys loaded) are out
            const bool diag = k0 + KT - 1 > pos0;
            const int lim = pos_row - k0 - half * HC;  // columns c <= lim are visible
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (diag) {
#pragma unroll
                for (int c = 0; c < HC; ++c) {
                    s[c] = c <= lim ? s[c] : -INFINITY;
                    m4[c & 3] = fmaxf(m4[c & 3], s[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < HC; ++c) m4[c & 3] = fmaxf(m4[c & 3], s[c]);
            }
            float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // row maximum over both halves
            red_s[j & 1][half][row] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xb[j & 1]);
            if (!mbar_wait(&xb[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            mx = fmaxf(mx, red_s[j & 1][half ^ 1][row]);
            const float mt = mx == -INFINITY ? -INFINITY : mx * qs;  // base-2 domain
            const bool move = mt > m_used + kPrefillRescaleLog2;
            float alpha = 1.f;
            if (move) {
                alpha = exp2_fast(m_used - mt);  // 0 on the first tile
                m_used = mt;
            }
            const float nm = -m_used;
            l *= alpha;
            if (j >= 1 && __any_sync(0xffffffffu, move)) {
                // rescale O: P_{j-1} V_{j-1} must be in it first
                if (!od_wait(j - 1)) {
                    ok = false;
                    break;
                }
                {
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        float o[32];
                        tmem_ld32(tl + kColO + half * HD + c * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_st32(tl + kColO + half * HD + c * 32, o);
                    }
                    tmem_wait_st();
                }
            }
            if (j == ntiles - 1) {
                // V rows of the last 16-key group past the context end are
                // unwritten pool slots: zero them (weight 0 times anything
                // must stay 0) once their tensor-map fill has landed
                const int z0 = L - k0, z1 = n16_last * 16;
                if (z0 < z1) {
                    const int sv = NH + j % NH;
                    if (!mbar_wait(&full[sv], (uint32_t)(j / NH) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    unsigned char *vs = ring + (size_t)sv * p.slot_bytes;
                    for (int i = sid; i < (z1 - z0) * NDC * 8; i += 32 * kPrefillSoftmaxWarps) {
                        const int r = z0 + i / (NDC * 8), c = i % (NDC * 8);
                        *reinterpret_cast<uint4 *>(vs + (c >> 3) * kSlotBlk + r * 128 + ((c & 7) << 4)) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            // ---- weights and P over S_j, 16 keys at a time: the chunk's S
            // columns are read back and its P parts written over them (high
            // parts in the first 8 columns, low parts in the next 8), so no
            // column is written before its S value is read (rolled loops:
            // small code for the warps that share a scheduler). ----
            float l4[2] = {0.f, 0.f};
            {
                const uint32_t hb = sb + half * HC;  // this half's 64 columns
                // one chunk; the causal mask only on tiles that reach the diagonal
                auto chunk = [&](int c, auto masked) {
                    float w[16];
                    tmem_ld16(hb + c * 16, w);
                    const int cl = lim - c * 16;
                    float2 l2 = make_float2(0.f, 0.f);
                    uint32_t pw[16];  // P high parts (words 0-7), low parts (words 8-15)
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 t = ffma2(make_float2(w[2 * i], w[2 * i + 1]), make_float2(qs, qs), make_float2(nm, nm));
                        float2 e = make_float2(exp2_fast(t.x), exp2_fast(t.y));
                        if constexpr (decltype(masked)::value) {
                            e.x = 2 * i <= cl ? e.x : 0.f;
                            e.y = 2 * i + 1 <= cl ? e.y : 0.f;
                        }
                        l2 = fadd2(l2, e);
                        Op::split_p(e.x, e.y, pw[i], pw[8 + i]);
                    }
                    l4[c & 1] += l2.x + l2.y;
                    tmem_st16u(hb + c * 16, pw);
                };
                if (diag) {
#pragma unroll 1
                    for (int c = 0; c < HC / 16; ++c) chunk(c, std::true_type{});
                } else {
#pragma unroll 1
                    for (int c = 0; c < HC / 16; ++c) chunk(c, std::false_type{});
                }
            }
            l += l4[0] + l4[1];
            // confirm P_{j-2} V_{j-2} (long done) before P_j is published: P_j V_j
            // could otherwise complete and put odone[j & 1] two phases ahead
            if (j >= 2 && !od_wait(j - 2)) {
                ok = false;
                break;
            }
            tmem_wait_st();
            fence_async_smem();  // V rows zeroed above
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[j & 1]);
        }
        if (ok && od_wait(ntiles - 1)) {  // the last product: every earlier one is done too
            // row sum over both halves
            red_s[ntiles & 1][half][row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xb[ntiles & 1]);
            ok = mbar_wait(&xb[ntiles & 1], (uint32_t)(ntiles >> 1) & 1u, abort_flag);
            if (ok) {
                // ---- normalise and store this half of the rows of real tokens ----
                const float inv = 1.f / (l + red_s[ntiles & 1][half ^ 1][row]);
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.out) + (grow + half * HD) * E);
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    float o[32];
                    tmem_ld32(tl + kColO + half * HD + c * 32, o);
                    if (valid) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[c * 4 + i] = make_uint4(Op::pack(o[8 * i] * inv, o[8 * i + 1] * inv),
                                                        Op::pack(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                                        Op::pack(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                                        Op::pack(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                    }
                }
            }
        } else {
            ok = false;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrefillTmemCols);
    }
}

}  // namespace pa
