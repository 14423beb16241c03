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
// Work decomposition: one CTA per (request, KV head, tile of 2 QT new
// tokens), as two query tiles A and B of QT tokens each.  A query tile's 128
// rows are its QT tokens x the G query heads of the KV head (row r = token
// r / G, head r % G), so every K/V tile staged in shared memory serves both
// query tiles and the whole head group.  The CTA streams keys 0 .. pos(last
// token of the tile) in tiles of 128 and masks, per row, the keys past the
// row's own position; query tile A stops at its own last position.  Every
// CTA ranks the (request, CTA tile) pairs by their key tiles, from the
// lengths, and takes the pair of its own rank: heavy pairs start first.
//
// Inside a CTA (5th-generation tensor cores, accumulators in tensor memory):
//   warps 0,10 producers of K and of V: each walks the block table (one tile
//              ahead) and fills its own ring of slots with tensor-map boxes
//              ([d-block][key][128 B], 128-byte swizzle: the canonical K-major
//              layout for K, MN-major for V);
//   warp 1     allocates tensor memory; one lane issues every tcgen05.mma,
//              alternating between the query tiles so that the tensor core
//              works on one while the softmax of the other runs:
//                S_t = Q_t K_j^T (M 128 rows, N 128 keys, into query tile t's
//                                 S buffer),
//                O_t += P_t V_j  (M 128 rows, N = D, K = keys; P read from
//                                 tensor memory, where the softmax wrote it
//                                 over S_t, in two 16-bit parts, high and
//                                 low, as in decode);
//   warps 2-9  softmax: warps 2-5 take query tile A, warps 6-9 query tile B,
//              one thread per row (tensor-memory lane = row, the warp's lane
//              quarter fixed by its index), so a row's maximum and sum never
//              leave the thread.  They copy their q rows into the swizzled Q
//              tile, then per key tile load the whole S row into registers
//              (one 128-column load), take its maximum, run the fp32 online
//              softmax in the base-2 domain, write P (high and low parts)
//              over S, and at the end read O, divide and store the row.
// The issuing lane keeps every operand descriptor in registers and adds
// offsets to it: the tensor core queues only a few products ahead, so the
// issuer's own latency between products is idle tensor time.
// The tensor pipe runs its products in issue order, so S_t of the next key
// tile (issued after P_t V_j) never overwrites P_t before it is read.  The
// running maximum is moved only when a tile's maximum exceeds it by more than
// 2^8 (weights stay below 256, exact in fp32 and safe in 16 bits); the
// rescale of O in tensor memory is then rare.  The final division uses the
// same maximum as every weight, so the result is the plain softmax.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace pa {

constexpr int kPrefillRows = 128;     // rows per query tile: M of every tensor-core product
constexpr int kPrefillQTiles = 2;     // query tiles per CTA, sharing every K/V tile
constexpr int kPrefillKT = 128;       // keys per tile: N of S, K of P V
constexpr int kPrefillSoftmaxWarps = 8;
constexpr int kPrefillVWarp = 2 + kPrefillSoftmaxWarps;             // the V producer
constexpr int kPrefillThreads = (3 + kPrefillSoftmaxWarps) * 32;  // K producer, MMA, softmax, V producer
constexpr int kPrefillTmemCols = 512; // S / P of both query tiles (2 x 128 columns) + O of both (2 x D)
constexpr int kPrefillMaxSlots = 8;   // K / V ring slots
constexpr float kPrefillRescaleLog2 = 8.f;
constexpr int kPrefillMaxRankedPairs = 2048;  // (request, CTA tile) pairs ranked in-kernel

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
    int32_t QT;          // new tokens per query tile (QT * G = kPrefillRows); a CTA takes 2 QT
    int32_t br_log2;     // rows of one box = min(kPrefillKT, bs)
    int32_t nslots;      // ring slots, even: K of tile j in slot j mod (nslots/2), V of tile j in the second half
    int32_t num_qtiles;  // CTA tiles of 2 QT tokens the grid covers per request
    uint32_t off_ring, slot_bytes;  // shared-memory layout (from the 1024-aligned base; Q tiles at 0)
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
    constexpr uint32_t kQTile = kPrefillRows * D * 2;  // one query tile in shared memory
    constexpr uint32_t kSlotBlk = KT * 128u;           // one d-block of a K / V slot
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescPV = umma_idesc(kPrefillRows, D, false, true, kBf16);
    constexpr uint32_t kColO = kPrefillQTiles * KT;    // tensor-memory column of O of query tile 0
    static_assert(kPrefillQTiles * (KT + D) <= kPrefillTmemCols, "tensor memory");
    static_assert(kBlk == kSlotBlk, "Q and K blocks share the k-step offsets");
    // At D = 64 the 512 columns leave 64 per query tile for the second half of P:
    // the next S can then go over the S buffer as soon as the first half's P V is
    // issued, while the softmax still computes the second half (it holds the
    // whole S row in registers from its one load).
    constexpr bool kP2Own = kPrefillQTiles * (KT + D) + kPrefillQTiles * (KT / 2) <= kPrefillTmemCols;
    constexpr uint32_t kColP2 = kPrefillQTiles * (KT + D);  // second-half P of query tile 0, when kP2Own
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw;  // the plan leaves no room to realign: checked below
    // mbarriers: full[], empty[] (ring), sfull[2] (per query tile), pfull[2][2] (per
    // query tile and half of the key tile), odone[2][2] (per query tile and key-tile
    // parity), qfull, fin
    constexpr int kOffSfull = 2 * kPrefillMaxSlots, kOffPfull = kOffSfull + 2;
    constexpr int kOffOdone = kOffPfull + 4, kOffQfull = kOffOdone + 4, kOffFin = kOffQfull + 1;
    constexpr int kBars = kOffFin + 1;
    __shared__ uint64_t bars[kBars];
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NH = p.nslots / 2;  // K slots 0 .. NH-1, V slots NH .. 2NH-1
    uint64_t *full = bars, *empty = bars + kPrefillMaxSlots;
    uint64_t *sfull = bars + kOffSfull;  // [query tile]: its S product done (one phase per key tile)
    uint64_t *pfull = bars + kOffPfull;  // [query tile][half]: P of keys 64h .. 64h+63 written
    uint64_t *odone = bars + kOffOdone;  // [query tile][key-tile parity]: P V product done
    uint64_t *qfull = bars + kOffQfull, *fin = bars + kOffFin;
    volatile int *abort_flag = &abort_s;

    if (smem_u32(smem_raw) & 1023u) {  // the 128-byte swizzle needs 1024-byte aligned tiles
        if (tid == 0) set_error(p.error, PA_DEVERR_SMEM);
        return;
    }
    // ---- the CTA's tile: request, KV head, new tokens [t0, t0 + ntok) ----
    // ---- the CTA's (request, CTA tile) pair: pairs ranked by their key tiles,
    // heaviest first, so the hardware's in-order dispatch of CTAs to free SMs
    // is a longest-first list schedule; the KV heads of a pair are consecutive ----
    const int g = (int)(blockIdx.x % (unsigned)p.Hkv);
    const int rank = (int)(blockIdx.x / (unsigned)p.Hkv);
    int pair;
    {
        const int npairs = p.B * p.num_qtiles;
        if (npairs <= kPrefillMaxRankedPairs) {
            __shared__ int hist[256];
            __shared__ uint8_t bucket_of[kPrefillMaxRankedPairs];
            __shared__ int pick;
            for (int i = tid; i < 256; i += kPrefillThreads) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < npairs; i += kPrefillThreads) {
                const int bb = i / p.num_qtiles, qq = i - bb * p.num_qtiles;
                const int Lb = p.context_lens[bb], nb = p.query_start[bb + 1] - p.query_start[bb];
                const int tt0 = qq * kPrefillQTiles * p.QT;
                int work = 0;  // key tiles of the pair's query tiles (0: no tokens, or a bad length)
                if (nb > tt0 && nb <= Lb && Lb <= p.max_blocks * p.bs) {
#pragma unroll
                    for (int t = 0; t < kPrefillQTiles; ++t) {
                        const int last = min(nb, tt0 + (t + 1) * p.QT);  // tokens up to the tile's last
                        if (last > tt0 + t * p.QT) work += (Lb - nb + last + KT - 1) / KT;
                    }
                }
                const int bk = work > 0 ? 1 + min(work, 254) : 0;
                bucket_of[i] = (uint8_t)bk;
                atomicAdd(&hist[bk], 1);
            }
            __syncthreads();
            if (warp == 0) {
                // lane l sums buckets 255 - 8l .. 248 - 8l; a prefix over the lanes gives
                // the pairs heavier than each lane's range
                int s8 = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) s8 += hist[255 - 8 * lane - k];
                int incl = s8;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                const int holder = __ffs(__ballot_sync(0xffffffffu, rank < incl)) - 1;
                int bk = 0, before = incl - s8;
                if (lane == holder) {
                    for (int k = 0; k < 8; ++k) {
                        const int c = hist[255 - 8 * lane - k];
                        if (rank < before + c) {
                            bk = 255 - 8 * lane - k;
                            break;
                        }
                        before += c;
                    }
                }
                bk = __shfl_sync(0xffffffffu, bk, holder);
                before = __shfl_sync(0xffffffffu, before, holder);
                // the (rank - before)-th pair of bucket bk, in index order
                int want = rank - before;
                for (int base = 0; base < npairs; base += 32) {
                    const int i = base + lane;
                    const bool hit = i < npairs && bucket_of[i] == bk;
                    const unsigned hm = __ballot_sync(0xffffffffu, hit);
                    const int c = __popc(hm);
                    if (want < c) {
                        if (hit && __popc(hm & ((1u << lane) - 1u)) == want) pick = i;
                        break;
                    }
                    want -= c;
                }
            }
            __syncthreads();
            pair = pick;
        } else {
            // too many pairs to rank: requests in order, each one's latest tiles first
            pair = (rank / p.num_qtiles) * p.num_qtiles + (p.num_qtiles - 1 - rank % p.num_qtiles);
        }
    }
    const int b = pair / p.num_qtiles, qt = pair - b * p.num_qtiles;
    const int cap = p.max_blocks * p.bs;
    const int L = p.context_lens[b];
    const int q0 = p.query_start[b];
    const int n = p.query_start[b + 1] - q0;
    if (L < 0 || L > cap || n < 0 || n > L || n > p.num_qtiles * kPrefillQTiles * p.QT) {
        if (tid == 0 && g == 0 && qt == 0) set_error(p.error, PA_DEVERR_CONTEXT_LEN);
        return;
    }
    const int t0 = qt * kPrefillQTiles * p.QT;
    if (t0 >= n) return;
    // query tile t: tokens t0 + t QT .. + ntok_t - 1 (ntok_t may be 0 for tile B)
    int ntok_q[kPrefillQTiles], nkt[kPrefillQTiles], n16_q[kPrefillQTiles];
#pragma unroll
    for (int t = 0; t < kPrefillQTiles; ++t) {
        ntok_q[t] = max(0, min(p.QT, n - (t0 + t * p.QT)));
        // keys 0 .. kend_t - 1 are visible to some row of query tile t
        const int kend_t = ntok_q[t] > 0 ? L - n + t0 + t * p.QT + ntok_q[t] : 0;
        nkt[t] = (kend_t + KT - 1) / KT;
        n16_q[t] = nkt[t] > 0 ? (kend_t - (nkt[t] - 1) * KT + 15) >> 4 : 0;  // 16-key groups of its last tile
    }
    const int ntiles = max(nkt[0], nkt[1]);  // key tiles the CTA streams
    const int kend = L - n + t0 + ntok_q[0] + ntok_q[1];

    if (tid == 0) {
        for (int s = 0; s < 2 * NH; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int t = 0; t < kPrefillQTiles; ++t) {
            mbar_init(&sfull[t], 1);
            for (int par = 0; par < 2; ++par) {
                mbar_init(&pfull[t * 2 + par], 4);  // the four warps of query tile t, per half
                mbar_init(&odone[t * 2 + par], 1);
            }
        }
        mbar_init(qfull, kPrefillSoftmaxWarps);
        mbar_init(fin, 1);
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
            const uint32_t r_addr = smem_u32(ring);
            // Operand descriptors are built once; a shared-memory offset (every
            // address here is below 256 KB) adds to the start-address field as
            // offset / 16, so each product below costs one add per operand.
            const uint64_t qdesc = umma_desc_sw128(smem_u32(smem), 16, 1024);        // Q tiles, K-major
            const uint64_t kdesc = umma_desc_sw128(r_addr, 16, 1024);                // K slots, K-major
            const uint64_t vdesc = umma_desc_sw128(r_addr, kSlotBlk, 1024);          // V slots, MN-major
            const uint32_t slot16 = p.slot_bytes >> 4;
            bool ok = mbar_wait(qfull, 0u, abort_flag);
            bool issued_any = false;
            // Everything a product needs is in registers before the loop: the
            // issuing thread's own latency between products is tensor-core idle
            // time, since the core queues only a few products ahead.
            const int nk0 = nkt[0], nk1 = nkt[1];
            const uint32_t idesc_full = umma_idesc(kPrefillRows, KT, false, false, kBf16);
            const uint32_t idesc_last0 = umma_idesc(kPrefillRows, n16_q[0] * 16, false, false, kBf16);
            const uint32_t idesc_last1 = umma_idesc(kPrefillRows, n16_q[1] * 16, false, false, kBf16);
            // S_t = Q_t K_j^T into query tile t's buffer (K of tile j in slot sk, fill
            // parity par); the last user of the K slot releases it
            auto s_issue = [&](auto tc, int j, int sk, uint32_t par) {
                constexpr int t = decltype(tc)::value;
                if (!ok) return;
                if (!mbar_wait(&full[sk], par, abort_flag)) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                const uint32_t idesc = j == (t ? nk1 : nk0) - 1 ? (t ? idesc_last1 : idesc_last0) : idesc_full;
                const uint64_t ad = qdesc + (uint64_t)(t * (kQTile >> 4));
                const uint64_t bd = kdesc + (uint64_t)(sk * slot16);
                const uint32_t ds = tmem + (uint32_t)t * KT;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    // k-step ks: 64-column block ks / 4 (16 KB apart), 32 bytes per step inside it
                    const uint32_t off = (uint32_t)((ks >> 2) * (kBlk >> 4) + (ks & 3) * 2);
                    umma_f16(ds, ad + off, bd + off, idesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&sfull[t]);
                // K slot j is read for the last time by the last query tile that sees tile j
                if (t == kPrefillQTiles - 1 || j >= nk1) umma_commit(&empty[sk]);
                issued_any = true;
            };
            // O_t += P_t V_j over keys 64h .. 64h+63 (each 16-key group: P high part,
            // then low part; V of tile j in slot NH + sk).  The softmax publishes P
            // in two halves, so the first half's products overlap the second
            // half's weights.  After the second half the last user of the V slot
            // releases it.
            auto pv = [&](auto tc, auto hc, int j, int sk, uint32_t par) {
                constexpr int t = decltype(tc)::value, h = decltype(hc)::value;
                if (!ok) return;
                const int sv = NH + sk;
                if (!mbar_wait(&pfull[t * 2 + h], (uint32_t)j & 1u, abort_flag) ||
                    (h == 0 && !mbar_wait(&full[sv], par, abort_flag))) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                const uint64_t bd = vdesc + (uint64_t)(sv * slot16);  // keys 16kk.. at +16kk rows of 128 B
                // P_t in its S buffer: keys 16kk .. 16kk+15 in columns 16kk .. 16kk+7
                // (high parts) and 16kk+8 .. 16kk+15 (low parts), two keys per column
                constexpr int kH = KT / 32;  // 16-key groups per half
                // A of group kk at column pa_off + 16 kk (the second half from its own columns when kP2Own)
                constexpr uint32_t pa_off = (kP2Own && h == 1) ? kColP2 + (uint32_t)(t * (KT / 2) - kH * 16)
                                                               : (uint32_t)t * KT;
                constexpr uint32_t od_off = kColO + (uint32_t)t * D;
                const uint32_t acc0 = j > 0 ? 1u : 0u;
                if (j != (t ? nk1 : nk0) - 1) {
#pragma unroll
                    for (int kk = h * kH; kk < (h + 1) * kH; ++kk) {
                        umma_f16_ts(tmem + od_off, tmem + pa_off + kk * 16, bd + (uint64_t)(kk * 128), kIdescPV,
                                    kk > 0 ? 1u : acc0);
                        umma_f16_ts(tmem + od_off, tmem + pa_off + kk * 16 + 8, bd + (uint64_t)(kk * 128), kIdescPV,
                                    1u);
                    }
                } else {
                    const int n16 = min(t ? n16_q[1] : n16_q[0], (h + 1) * kH);
                    for (int kk = h * kH; kk < n16; ++kk) {
                        umma_f16_ts(tmem + od_off, tmem + pa_off + kk * 16, bd + (uint64_t)(kk * 128), kIdescPV,
                                    kk > 0 ? 1u : acc0);
                        umma_f16_ts(tmem + od_off, tmem + pa_off + kk * 16 + 8, bd + (uint64_t)(kk * 128), kIdescPV,
                                    1u);
                    }
                }
                if (h == 1) {
                    umma_commit(&odone[t * 2 + (j & 1)]);
                    if (t == kPrefillQTiles - 1 || j >= nk1) umma_commit(&empty[sv]);
                }
                issued_any = true;
            };
            using T0 = std::integral_constant<int, 0>;
            using T1 = std::integral_constant<int, 1>;
            auto pv_both = [&](auto tc, int j, int sk, uint32_t par) {
                pv(tc, T0{}, j, sk, par);
                pv(tc, T1{}, j, sk, par);
            };
            static_assert(kPrefillQTiles == 2, "the issue order below names the two query tiles");
            // ring position of tile j (slot j mod NH, fill parity (j / NH) & 1) and of tile j + 1
            int sc = 0, sn = NH > 1 ? 1 : 0;
            uint32_t pc = 0u, pn = NH > 1 ? 0u : 1u;
            if (nk0 > 0) s_issue(T0{}, 0, sc, pc);
            if (nk1 > 0) s_issue(T1{}, 0, sc, pc);
            // alternate between the query tiles: while one tile's softmax runs, the
            // tensor core takes the other tile's P V and next S
            for (int j = 0; j < ntiles && ok; ++j) {
                if constexpr (kP2Own) {
                    // first half's P V, the next S over the S buffer, then the second half's P V
                    if (j < nk0) {
                        pv(T0{}, T0{}, j, sc, pc);
                        if (j + 1 < nk0) s_issue(T0{}, j + 1, sn, pn);
                        pv(T0{}, T1{}, j, sc, pc);
                    }
                    if (j < nk1) {
                        pv(T1{}, T0{}, j, sc, pc);
                        if (j + 1 < nk1) s_issue(T1{}, j + 1, sn, pn);
                        pv(T1{}, T1{}, j, sc, pc);
                    }
                } else {
                    if (j < nk0) {
                        pv_both(T0{}, j, sc, pc);
                        if (j + 1 < nk0) s_issue(T0{}, j + 1, sn, pn);
                    }
                    if (j < nk1) {
                        pv_both(T1{}, j, sc, pc);
                        if (j + 1 < nk1) s_issue(T1{}, j + 1, sn, pn);
                    }
                }
                sc = sn;
                pc = pn;
                if (++sn == NH) {
                    sn = 0;
                    pn ^= 1u;
                }
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
        // ================= softmax: one thread per row =================
        constexpr int HD = D;                 // O columns per thread
        const int qtile = (warp - 2) >> 2;    // query tile of this warp
        const int quad = warp & 3;            // tensor-memory lane quarter of this warp
        const int row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);  // this warp's lanes
        const uint32_t sb = tl + (uint32_t)qtile * KT;             // S / P of this query tile
        const uint32_t ob = tl + kColO + (uint32_t)qtile * D;      // O of this query tile
        uint64_t *pf = pfull + qtile * 2, *odn = odone + qtile * 2;
        const int tok = row >> p.g_log2, hj = row & (p.G - 1);
        const int ntok = qtile ? ntok_q[1] : ntok_q[0];
        const int n16_last = qtile ? n16_q[1] : n16_q[0];  // 16-key groups of the tile's last key tile
        const int tq0 = t0 + qtile * p.QT;    // first new token of this query tile
        const bool valid = tok < ntok;
        const size_t grow = ((size_t)(q0 + tq0 + tok) * p.Hq + (size_t)g * p.G + hj) * D;  // q / out row
        // ---- Q tile: row `row`, K-major with the 128-byte swizzle ----
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(p.q) + grow * E);
            unsigned char *qs = smem + (size_t)qtile * kQTile;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (valid) {
                    v = __ldg(src + c);
                    v.x ^= p.qflip;
                    v.y ^= p.qflip;
                    v.z ^= p.qflip;
                    v.w ^= p.qflip;
                }
                *reinterpret_cast<uint4 *>(qs + (c >> 3) * kBlk + row * 128 + (((c & 7) ^ (row & 7)) << 4)) = v;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        const int nj = qtile ? nkt[1] : nkt[0];
        const int pos0 = L - n + tq0;                               // position of the query tile's first token
        const int pos_row = pos0 + (valid ? tok : max(ntok, 1) - 1);  // rows past the tokens mirror the last token
        const float qs = p.qscale;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        // P V completions, confirmed per barrier in order: odone[j & 1] phase
        // j >> 1 is P_j V_j, and P_{j+2} V_{j+2} cannot complete before the
        // softmax of tile j+2 has run, so a parity wait never skips a phase
        int od_next[2] = {0, 0};
        auto od_wait = [&](int i) {
            int &nx = od_next[i & 1];
            for (; nx <= (i >> 1); ++nx)
                if (!mbar_wait(&odn[i & 1], (uint32_t)nx & 1u, abort_flag)) return false;
            tc_fence_after();
            return true;
        };
        for (int j = 0; j < nj; ++j) {
            const int k0 = j * KT;
            if (!mbar_wait(&sfull[qtile], (uint32_t)j & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // keys past the row's position (or past the keys loaded) are out
            const bool diag = k0 + KT - 1 > pos0;
            const int lim = pos_row - k0;  // columns c <= lim are visible
            // ---- the whole S row in registers (one load, one wait); masked keys
            // become -inf, so their weights below come out 0 ----
            float sr[KT];
            tmem_ld128(sb, sr);
            if (diag) {
#pragma unroll
                for (int c = 0; c < KT; ++c) sr[c] = c <= lim ? sr[c] : -INFINITY;
            }
            float mx;
            {
                float m4[4] = {sr[0], sr[1], sr[2], sr[3]};
#pragma unroll
                for (int c = 4; c < KT; c += 8)
#pragma unroll
                    for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], sr[c + i], sr[c + 4 + i]);
                mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
            }
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
#pragma unroll 1
                for (int c = 0; c < HD / 16; ++c) {
                    float o[16];
                    tmem_ld16(ob + c * 16, o);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(o[i] * alpha);
                    tmem_st16u(ob + c * 16, w);
                }
                tmem_wait_st();
            }
            if (j == nj - 1) {
                // V rows of the last 16-key groups this tile's P V product reads that
                // lie past the context end are unwritten pool rows: zero them
                // (weight 0 times anything must stay 0) once their fill has landed
                const int z0 = max(0, L - k0), z1 = n16_last * 16;
                if (z0 < z1) {
                    const int sv = NH + j % NH;
                    if (!mbar_wait(&full[sv], (uint32_t)(j / NH) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    unsigned char *vs = ring + (size_t)sv * p.slot_bytes;
                    for (int i = quad * 32 + lane; i < (z1 - z0) * NDC * 8; i += 128) {
                        const int r = z0 + i / (NDC * 8), c = i % (NDC * 8);
                        *reinterpret_cast<uint4 *>(vs + (c >> 3) * kSlotBlk + r * 128 + ((c & 7) << 4)) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            // confirm P_{j-2} V_{j-2} (long done) before P_j is published: P_j V_j
            // could otherwise complete and put odone[j & 1] two phases ahead
            if (j >= 2 && !od_wait(j - 2)) {
                ok = false;
                break;
            }
            // ---- weights, written over S as P in 16-key groups: high parts of
            // keys 16c .. 16c+15 in columns 16c .. 16c+7, low parts in 16c+8 ..
            // 16c+15; each half of the tile is published as soon as it is written ----
            float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            {
                const float2 qs2 = make_float2(qs, qs), nm2 = make_float2(nm, nm);
                const int nch = j == nj - 1 ? n16_last : KT / 16;  // 16-key groups the P V product reads
#pragma unroll
                for (int c = 0; c < KT / 16; ++c) {
                    if (kP2Own && c == KT / 32 && j >= 1 && c < nch && !od_wait(j - 1))
                        ok = false;  // the second half's columns are free once P_{j-1} V_{j-1} is done
                    if (c < nch) {
                        uint32_t pw[16];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 t = ffma2(make_float2(sr[16 * c + 2 * i], sr[16 * c + 2 * i + 1]), qs2, nm2);
                            const float2 e = make_float2(exp2_fast(t.x), exp2_fast(t.y));
                            l2[i & 1] = fadd2(l2[i & 1], e);
                            Op::split_p2(e, pw[i], pw[8 + i]);
                        }
                        if (kP2Own && c >= KT / 32)
                            tmem_st16u(tl + kColP2 + (uint32_t)(qtile * (KT / 2) + (c - KT / 32) * 16), pw);
                        else
                            tmem_st16u(sb + c * 16, pw);
                    }
                    if (c == KT / 32 - 1 || c == KT / 16 - 1) {
                        tmem_wait_st();
                        if (c == KT / 32 - 1) fence_async_smem();  // V rows zeroed above
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&pf[c == KT / 16 - 1 ? 1 : 0]);
                    }
                }
            }
            l += (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
            if (!ok) break;
        }
        if (ok && nj > 0 && od_wait(nj - 1)) {  // the last product: every earlier one is done too
            // ---- normalise and store the row (real tokens only) ----
            const float inv = 1.f / l;
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.out) + grow * E);
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                float o[32];
                tmem_ld32(ob + c * 32, o);
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[c * 4 + i] = make_uint4(Op::pack(o[8 * i] * inv, o[8 * i + 1] * inv),
                                                    Op::pack(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                                    Op::pack(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                                    Op::pack(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                }
            }
        } else if (nj > 0) {
            ok = false;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) set_error(p.error, PA_DEVERR_TIMEOUT);
        }
    }
    // Every warp reaches the CTA barrier whole: one lane of warp 1 issued the
    // products while the others went ahead, and a barrier met by part of a warp
    // does not hold the rest of the CTA (tensor memory must outlive the last
    // read of O).
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPrefillTmemCols);
    }
}

}  // namespace pa
