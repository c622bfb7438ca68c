// Absorbed-MLA decode attention over the packed 2-bit cache ("RoLaQ", §2.1, §3.3) with
// both tensor-core A operands in tensor memory.
//
// rolaq_decode_tm: one CTA per (work item, 16 query heads); the item's pages are taken
// two at a time as 128-token tiles.  For a tile the decoded content latent x (fp16) is
// written into tensor memory twice:
//   token-major    lanes = the tile's 128 tokens, columns = the 512 channels (in slot
//                  order, two per column): the A operand of QK (M = 128 tokens, N = 16
//                  heads, K = 512), reused by the tensor cores without any shared-memory
//                  traffic;
//   channel-major  for every channel group, lanes = its 128 channels, columns = 64 tokens
//                  of one page: the A operand of PV (M = 128 channels, N = 16 heads,
//                  K = tokens), one 32-column slot per group.
// A tensor-core product with A in tensor memory costs about N/2 cycles, four times less
// than with A read from shared memory at N = 16, and x never passes through shared memory.
//
// Warp roles (19 warps):
//   warp 0        producer: per tile, two bulk tensor copies per page (codes + metadata
//                 rows into the page stage, RoPE-key rows into a 128-row key tile), four
//                 stages;
//   warp 1        QK issue: 32 fp16 products from the token-major x and 4 bf16 products
//                 for the RoPE keys (read from shared memory) into S;
//   warp 18       PV issue: 16 products per page from the channel-major x into O;
//   warps 2..5    softmax: thread = token (S lane); the running maximum per head moves
//                 only when a score exceeds it by more than 2^8 (a vote among the four
//                 warps); the fp16 probabilities go to shared memory as the MN-major B
//                 operand;
//   warps 6..13   token-major x, two per tensor-memory lane quarter (channel groups 0-1
//                 and 2-3): thread (token, group) forms the four fp16 values mean +
//                 scale * level of its (token, group) and turns each code into x with one
//                 PRMT per pair; it also leaves the (token, group)'s fp16 scale and mean
//                 in a per-tile table;
//   warps 14..21  channel-major x, two per lane quarter: thread (code byte, four tokens)
//                 gathers the byte of four tokens, looks the four fp16 levels up with one
//                 PRMT per token pair and applies the pair's (scale, mean) from the table
//                 with one fp16x2 FMA.  Its slots form a five-deep ring (one slot = one
//                 group x one page), and each slot's stores complete while the next slot
//                 is computed.
// The merge of the work items is rolaq_decode_merge.
#pragma once
#include "decode.cuh"

namespace rolaq {

constexpr int kTmThreads = 608;
constexpr int kTmTok = 128;                          // tokens per tile (two pages)
constexpr int kTmStages = 4;
constexpr int kTmHeads = 16;
constexpr int kTmTm0 = 2;                            // token-major warps 2..9 (2..5 also softmax)
constexpr int kTmCm0 = 10;                           // channel-major warps 10..17
constexpr int kTmPv = 18;                            // PV issue warp
constexpr int kTmCmRows = 80;                        // page rows 0..79: codes, metadata
constexpr int kTmKrRows = 64;                        // page rows 80..143: RoPE keys
constexpr uint32_t kTmColXq = 0;                     // token-major x: 256 columns
constexpr uint32_t kTmColS = 256;                    // scores: two tiles x 16 heads
constexpr uint32_t kTmColO = 288;                    // O: 4 groups x 16 heads
constexpr uint32_t kTmColXp = 352;                   // channel-major x: ring of 5 slots x 32 columns
constexpr int kTmXpSlots = 5;
constexpr uint32_t kTmCols = 512;
// instruction descriptors: fp32 accumulate, M = 128, N = 16
constexpr uint32_t kTmIdQk = (1u << 4) | ((uint32_t)(kTmHeads >> 3) << 17) | ((128u >> 4) << 24);   // f16
constexpr uint32_t kTmIdRope = kTmIdQk | (1u << 7) | (1u << 10);                                     // bf16
constexpr uint32_t kTmIdPv = kTmIdQk | (1u << 16);                                                   // B MN-major

struct TmSmem {
    alignas(1024) uint8_t cm[kTmStages][2][kTmCmRows * 128];   // codes + metadata, per page
    alignas(1024) uint8_t kr[kTmStages][kTmTok * 128];          // RoPE keys of both pages
    alignas(1024) uint8_t qc[kTmHeads * ROLAQ_D_C * 2];         // fp16 query (slot order), QK B
    alignas(128) uint8_t qr[kTmHeads * ROLAQ_D_R * 2];          // bf16 RoPE query
    alignas(1024) uint8_t P[2][kTmTok * 32];                    // fp16 probabilities, PV B
    uint4 tbl[3][ROLAQ_GROUPS][kTmTok / 4];                     // fp16x2 (sc01, sc23, mu01, mu23)
    float red[2][4][kTmHeads / 2];
    float mref[kTmHeads];
    float alpha[kTmHeads];
    int vote[2][2][4];
    alignas(8) uint64_t full[kTmStages];
    uint64_t pfree[kTmStages];
    uint64_t xq_full[2], xq_free[2];       // token-major x, channel groups 0-1 / 2-3
    uint64_t tbl_full[3], tbl_free[3];
    uint64_t xp_full[kTmXpSlots], xp_free[kTmXpSlots];
    uint64_t sfull[2], sfree[2], pready[2], pvdone[2];
    uint32_t tmem_base;
    int plan[4];
    int abort;
};
static_assert(sizeof(TmSmem) + 1024 <= 227 * 1024, "decode shared memory");

// Whether page `pg` (0-based within the item) of request b exists and is inside the pool.
__device__ __forceinline__ bool tm_page_ok(const DecodeArgs& args, int b, int first_page, int T, int pg) {
    return pg < T && page_ok(args, page_id(args, b, first_page + pg));
}

// Sixteen codes of one token (one 32-bit word, code j of byte b at bits 2j) into fp16
// pairs: r[k][0] = (x of byte 0's code k, x of byte 1's code k), r[k][1] the same for
// bytes 2 and 3.  The lookup pair (lo, hi) holds the low and high bytes of the token's
// four fp16 values, so a PRMT selector with nibbles (c, c + 4) picks value c: one
// multiply-add forms the selectors of four codes, the second pair uses its upper half.
__device__ __forceinline__ void tm_codes_to_x(uint32_t w, uint2 lut, uint32_t (&r)[4][2]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t m = (w >> (2 * k)) & 0x03030303u;
        const uint32_t sel = m * 0x11u + 0x40404040u;
        r[k][0] = prmt(lut.x, lut.y, sel);
        r[k][1] = prmt(lut.x, lut.y, sel >> 16);
    }
}

// Token-major x of one (token, group), streamed into tensor memory 32 channels at a time
// (16 columns of fp16 pairs in slot order per store), and the fp16 scale and mean of the
// (token, group) for the channel-major pass (both zero for tokens that take no 2-bit
// value).  `pg` is the page's stage (codes rows 0..63, metadata rows 64..79, 128-byte
// swizzle), `row` the token's row, `taddr` the token's lane at the group's first column.
__device__ __forceinline__ void tm_token_store(const uint8_t* pg, int row, int g, bool valid, bool prot,
                                               const __nv_bfloat16* prow, float la, float lb, uint32_t taddr,
                                               uint32_t& sc16, uint32_t& mu16) {
    uint2 lut = make_uint2(0u, 0u);
    uint4 cw0 = make_uint4(0u, 0u, 0u, 0u), cw1 = cw0;
    sc16 = 0u;
    mu16 = 0u;
    if (valid) {
        const float2 ms = *reinterpret_cast<const float2*>(pg + swz128(kMetaRow + (row >> 2), (row & 3) * 32 + 8 * g));
        if (!(fabsf(ms.x) + fabsf(ms.y) * lb < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        const uint32_t w01 = pack_f16(fmaf(ms.y, -lb, ms.x), fmaf(ms.y, -la, ms.x));
        const uint32_t w23 = pack_f16(fmaf(ms.y, la, ms.x), fmaf(ms.y, lb, ms.x));
        lut.x = prmt(w01, w23, 0x6420u);
        lut.y = prmt(w01, w23, 0x7531u);
        if (!prot) {
            const uint32_t sm2 = pack_f16(ms.y, ms.x);
            sc16 = sm2 & 0xFFFFu;
            mu16 = sm2 >> 16;
        }
        cw0 = *reinterpret_cast<const uint4*>(pg + row * 128 + (((2 * g) ^ (row & 7)) << 4));
        cw1 = *reinterpret_cast<const uint4*>(pg + row * 128 + (((2 * g + 1) ^ (row & 7)) << 4));
    }
    const uint32_t cw[8] = {cw0.x, cw0.y, cw0.z, cw0.w, cw1.x, cw1.y, cw1.z, cw1.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t v[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t r[4][2];
            tm_codes_to_x(cw[2 * c + h], lut, r);
#pragma unroll
            for (int k = 0; k < 4; ++k) { v[8 * h + k] = r[k][0]; v[8 * h + 4 + k] = r[k][1]; }
        }
        if (prot) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int w = 2 * c + h;
                const uint4 u0 = reinterpret_cast<const uint4*>(prow + 128 * g + 16 * w)[0];
                const uint4 u1 = reinterpret_cast<const uint4*>(prow + 128 * g + 16 * w)[1];
                const uint32_t pv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float a0 = (k & 1) ? bf16_hi(pv[k >> 1]) : bf16_lo(pv[k >> 1]);
                    const float a1 = (k & 1) ? bf16_hi(pv[2 + (k >> 1)]) : bf16_lo(pv[2 + (k >> 1)]);
                    const float b0 = (k & 1) ? bf16_hi(pv[4 + (k >> 1)]) : bf16_lo(pv[4 + (k >> 1)]);
                    const float b1 = (k & 1) ? bf16_hi(pv[6 + (k >> 1)]) : bf16_lo(pv[6 + (k >> 1)]);
                    v[8 * h + k] = pack_f16(a0, a1);
                    v[8 * h + 4 + k] = pack_f16(b0, b1);
                }
            }
        }
        tmem_st16(taddr + 16 * c, v);
    }
}

__global__ void __launch_bounds__(kTmThreads, 1)
rolaq_decode_tm(const __grid_constant__ CUtensorMap map_cm, const __grid_constant__ CUtensorMap map_kr,
                const DecodeArgs args) {
    extern __shared__ uint8_t smem_raw[];
    TmSmem& sm = *reinterpret_cast<TmSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hc = blockIdx.y;                 // 16-head chunk

    if (warp == 0) {
        PlanInfo pi = plan_lookup(args.seq_lens, args.batch, args.target_items, (int)blockIdx.x, -1);
        if (lane == 0) {
            sm.plan[0] = pi.b;
            sm.plan[1] = pi.first_page;
            sm.plan[2] = pi.n_pages;
        }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kTmStages; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.pfree[s]), 8 + 8 + 1);      // expansion warps + RoPE MMAs
        }
        for (int hx = 0; hx < 2; ++hx) {
            mbar_init(smem_u32(&sm.xq_full[hx]), 4);
            mbar_init(smem_u32(&sm.xq_free[hx]), 1);
        }
        for (int k3 = 0; k3 < 3; ++k3) {
            mbar_init(smem_u32(&sm.tbl_full[k3]), 8);
            mbar_init(smem_u32(&sm.tbl_free[k3]), 8);
        }
        for (int sl = 0; sl < kTmXpSlots; ++sl) {
            mbar_init(smem_u32(&sm.xp_full[sl]), 4);
            mbar_init(smem_u32(&sm.xp_free[sl]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&sm.sfull[s]), 1);
            mbar_init(smem_u32(&sm.sfree[s]), 8);
            mbar_init(smem_u32(&sm.pready[s]), 8);
            mbar_init(smem_u32(&sm.pvdone[s]), 1);
        }
        for (int h = 0; h < kTmHeads; ++h) sm.mref[h] = -INFINITY;
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_cm);
        prefetch_tmap(&map_kr);
    }
    __syncthreads();
    const int b = sm.plan[0];
    if (b < 0) return;                         // item past the end of the plan
    const int first_page = sm.plan[1], T = sm.plan[2];
    const int nt = (T + 1) >> 1;
    const int L = args.seq_lens[b];
    const int h0 = hc * kTmHeads;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&sm.tmem_base)), "r"(kTmCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // queries as B operands: fp16 content query in slot order, bf16 RoPE query
    {
        const uint16_t* qb = reinterpret_cast<const uint16_t*>(args.q + ((size_t)b * args.heads + h0) * ROLAQ_D_C);
        float qmax = 0.f;
        for (int e = threadIdx.x; e < kTmHeads * ROLAQ_D_C / 2; e += kTmThreads) {
            const int n = e / (ROLAQ_D_C / 2), s = 2 * (e % (ROLAQ_D_C / 2));
            const float v0 = __uint_as_float((uint32_t)qb[n * ROLAQ_D_C + slot_channel(s)] << 16);
            const float v1 = __uint_as_float((uint32_t)qb[n * ROLAQ_D_C + slot_channel(s + 1)] << 16);
            qmax = fmaxf(qmax, fmaxf(fabsf(v0), fabsf(v1)));
            *reinterpret_cast<uint32_t*>(sm.qc + plain_off(n, s, 64 * 128)) = pack_f16(v0, v1);
        }
        if (!(qmax < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        const uint32_t* rb = reinterpret_cast<const uint32_t*>(args.qr + ((size_t)b * args.heads + h0) * ROLAQ_D_R);
        for (int e = threadIdx.x; e < kTmHeads * ROLAQ_D_R / 2; e += kTmThreads) {
            const int n = e / (ROLAQ_D_R / 2), k = 2 * (e % (ROLAQ_D_R / 2));
            *reinterpret_cast<uint32_t*>(sm.qr + plain_off(n, k, 8 * 128)) = rb[e];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lane quarter

    if (warp == 0) {
        // ------------------------------------------------------------ producer ----
        if (lane == 0)
            for (int i = 0; i < nt; ++i) {
                const int st = i % kTmStages;
                if (i >= kTmStages)
                    mbar_wait(smem_u32(&sm.pfree[st]), (unsigned)((i / kTmStages - 1) & 1), &sm.abort);
                long long pid[2];
                bool ok[2];
                unsigned bytes = 0;
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int pg = 2 * i + p;
                    pid[p] = pg < T ? page_id(args, b, first_page + pg) : -1;
                    ok[p] = pg < T && page_ok(args, pid[p]);
                    if (pg < T && !ok[p]) raise_status(ROLAQ_STATUS_BAD_PAGE);
                    if (ok[p]) bytes += ROLAQ_PAGE_BYTES;
                }
                const uint32_t bar = smem_u32(&sm.full[st]);
                mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    if (ok[p]) {
                        tma_load_2d(smem_u32(sm.cm[st][p]), &map_cm, 0, (int)(pid[p] * kPageRows), bar);
                        tma_load_2d(smem_u32(sm.kr[st]) + p * kTmKrRows * 128, &map_kr, 0,
                                    (int)(pid[p] * kPageRows + kTmCmRows), bar);
                    }
            }
    } else if (warp == 1) {
        // ------------------------------------------------------------- QK issue ----
        const uint64_t dq = smem_desc(smem_u32(sm.qc), 128, 64 * 128, 0);
        const uint64_t dqr = smem_desc(smem_u32(sm.qr), 128, 8 * 128, 0);
        const uint64_t dkr = smem_desc(smem_u32(sm.kr[0]), 16, 1024, 2);
        for (int i = 0; i < nt; ++i) {
            {
                const int bi = i & 1, st = i % kTmStages;
                const uint32_t d = tmem + kTmColS + kTmHeads * bi;
                if (i >= 2) mbar_wait(smem_u32(&sm.sfree[bi]), (unsigned)(((i - 2) >> 1) & 1), &sm.abort);
                // the two halves of x (channel groups 0-1, 2-3) in the order they are
                // written; the first initialises S, the second adds the RoPE keys
                const int first = mbar_wait_either(smem_u32(&sm.xq_full[0]), smem_u32(&sm.xq_full[1]),
                                                   (unsigned)(i & 1), &sm.abort);
                const int hf0 = first < 0 ? 0 : first, hf1 = 1 - hf0;
                __syncwarp();
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < ROLAQ_D_C / 32; ++kk)
                        umma_ts1(d, tmem + kTmColXq + 8 * (16 * hf0 + kk),
                                 dq + (uint64_t)(((16 * hf0 + kk) * 256) >> 4), kTmIdQk, kk > 0 ? 1u : 0u);
                    umma_commit(smem_u32(&sm.xq_free[hf0]));
                }
                __syncwarp();
                mbar_wait(smem_u32(&sm.xq_full[hf1]), (unsigned)(i & 1), &sm.abort);
                mbar_wait(smem_u32(&sm.full[st]), (unsigned)((i / kTmStages) & 1), &sm.abort);
                __syncwarp();
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < ROLAQ_D_C / 32; ++kk)
                        umma_ts1(d, tmem + kTmColXq + 8 * (16 * hf1 + kk),
                                 dq + (uint64_t)(((16 * hf1 + kk) * 256) >> 4), kTmIdQk, 1u);
                    const uint64_t dk = dkr + (uint64_t)((st * kTmTok * 128) >> 4);
#pragma unroll
                    for (int kk = 0; kk < ROLAQ_D_R / 16; ++kk)
                        umma_ss1(d, dk + (uint64_t)((kk * 32) >> 4), dqr + (uint64_t)((kk * 256) >> 4), kTmIdRope, 1u);
                    umma_commit(smem_u32(&sm.sfull[bi]));
                    umma_commit(smem_u32(&sm.xq_free[hf1]));
                    umma_commit(smem_u32(&sm.pfree[st]));
                }
                __syncwarp();
            }
        }
    } else if (warp == kTmPv) {
        // ------------------------------------------------------------- PV issue ----
        // Its own warp, so PV of a tile never waits behind the next tile's QK: the two
        // streams touch different accumulators and operands, and each issuing thread's
        // commits track only its own products.
        const uint64_t dp = smem_desc_sw32(smem_u32(sm.P[0]), 256);
        auto pv = [&](int j) {
            const int bj = j & 1;
            mbar_wait(smem_u32(&sm.pready[bj]), (unsigned)((j >> 1) & 1), &sm.abort);
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int g = 0; g < ROLAQ_GROUPS; ++g) {
                    const int n = 8 * j + 4 * h + g, sl = n % kTmXpSlots;     // unit n of the x ring
                    mbar_wait(smem_u32(&sm.xp_full[sl]), (unsigned)((n / kTmXpSlots) & 1), &sm.abort);
                    __syncwarp();
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_ts1(tmem + kTmColO + 16 * g, tmem + kTmColXp + 32 * sl + 8 * kk,
                                     dp + (uint64_t)((bj * kTmTok * 32 + h * 2048 + kk * 512) >> 4), kTmIdPv,
                                     (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(smem_u32(&sm.xp_free[sl]));
                        if (h == 1 && g == ROLAQ_GROUPS - 1) umma_commit(smem_u32(&sm.pvdone[bj]));
                    }
                    __syncwarp();
                }
            }
        };
        for (int j = 0; j < nt; ++j) pv(j);
    } else if (warp >= kTmCm0) {
        // ------------------------------------------------ channel-major expansion ----
        const int q = warp & 3;                // TMEM lane quarter
        const int set = (warp - kTmCm0) >> 2;  // channel groups 2 set, 2 set + 1
        const float la = args.level_a, lb = args.level_b;
        const bool protect = args.n_sink > 0 || args.n_recent > 0;
        const int nslot = args.n_sink + args.n_recent;
        const int recent0 = L - args.n_recent;
        // fp16 levels (-b, -a, a, b): bytes 0-3 and 4-7 of the lookup pair
        const uint32_t lt0 = pack_f16(-lb, -la), lt1 = pack_f16(la, lb);
        // thread: code byte 32 g + 8 q + r (channels 4 (8 q + r) + s), tokens 16 m + 4 k + e
        const int r = lane >> 2, k = lane & 3;
        // A unit's tensor-memory stores complete in the background: they are waited for
        // (and the unit's barrier arrived on) only after the next unit has been computed.
        int pend_n = -1;
        auto flush = [&]() {
            if (pend_n >= 0) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_lane0(smem_u32(&sm.xp_full[pend_n % kTmXpSlots]));
                pend_n = -1;
            }
        };
        for (int j = 0; j < nt; ++j) {
            const int st = j % kTmStages;
            mbar_wait(smem_u32(&sm.full[st]), (unsigned)((j / kTmStages) & 1), &sm.abort);
            mbar_wait(smem_u32(&sm.tbl_full[j % 3]), (unsigned)((j / 3) & 1), &sm.abort);
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const uint8_t* pg = sm.cm[st][h];
                const int page_pos0 = (first_page + 2 * j + h) * kPageTok;
                const bool any_prot = protect && 2 * j + h < T && page_pos0 < L &&
                                      (page_pos0 < args.n_sink || page_pos0 + kPageTok > recent0);
#pragma unroll 1
                for (int gi = 0; gi < 2; ++gi) {
                    const int g = 2 * set + gi;
                    const int beta = 32 * g + 8 * q + r;
                    const uint32_t bsel = (uint32_t)(beta & 3) | ((uint32_t)((beta & 3) + 4) << 4);
                    uint32_t wv[4][4];
                    uint4 e4[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int row = 16 * m + 4 * k + e;
                            wv[m][e] = *reinterpret_cast<const uint32_t*>(pg + row * 128 + ((((beta >> 4) ^ row) & 7) << 4) +
                                                                          (beta & 12));
                        }
                        e4[m] = sm.tbl[j % 3][g][16 * h + 4 * m + k];
                    }
                    uint32_t xo[2][4][4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int row0 = 16 * m + 4 * k;
                        const uint32_t R = prmt(prmt(wv[m][0], wv[m][1], bsel), prmt(wv[m][2], wv[m][3], bsel), 0x5410u);
#pragma unroll
                        for (int s = 0; s < 4; ++s) {
                            const uint32_t m4 = (R >> (2 * s)) & 0x03030303u;
                            const uint32_t sel = m4 * 0x22u + 0x10101010u;
                            uint32_t x01 = hfma2(prmt(lt0, lt1, sel), e4[m].x, e4[m].z);
                            uint32_t x23 = hfma2(prmt(lt0, lt1, sel >> 16), e4[m].y, e4[m].w);
                            if (any_prot) {
                                // protected tokens of the quad take the bf16 side-store value
                                const int ch = 128 * g + 32 * q + 4 * r + s;
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int p = page_pos0 + row0 + e;
                                    if (p < L && (p < args.n_sink || p >= recent0)) {
                                        const int slot = p < args.n_sink ? p : args.n_sink + p % args.n_recent;
                                        const float v = __bfloat162float(args.prot[((size_t)b * nslot + slot) * ROLAQ_D_C + ch]);
                                        const uint32_t hv = pack_f16(v, v) & 0xFFFFu;
                                        uint32_t& xr = (e < 2) ? x01 : x23;
                                        xr = (e & 1) ? ((xr & 0xFFFFu) | (hv << 16)) : ((xr & 0xFFFF0000u) | hv);
                                    }
                                }
                            }
                            xo[s >> 1][m][2 * (s & 1)] = x01;
                            xo[s >> 1][m][2 * (s & 1) + 1] = x23;
                        }
                    }
                    flush();
                    const int n = 8 * j + 4 * h + g, sl = n % kTmXpSlots;     // unit n of the x ring
                    if (n >= kTmXpSlots)
                        mbar_wait(smem_u32(&sm.xp_free[sl]), (unsigned)((n / kTmXpSlots + 1) & 1), &sm.abort);
                    __syncwarp();
                    tc_fence_after();
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk)
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            tmem_st16x256(tmem + lane_base + ((uint32_t)(16 * blk) << 16) + kTmColXp + 32 * sl + 8 * m,
                                          xo[blk][m][0], xo[blk][m][1], xo[blk][m][2], xo[blk][m][3]);
                    pend_n = n;
                }
            }
            __syncwarp();
            mbar_arrive_lane0(smem_u32(&sm.pfree[st]));
            mbar_arrive_lane0(smem_u32(&sm.tbl_free[j % 3]));
        }
        flush();
    } else if (warp >= kTmTm0) {
        // -------------------------------------------------- token-major expansion ----
        const int q = warp & 3;                // TMEM lane quarter
        const int set = (warp - kTmTm0) >> 2;  // channel groups 2 set, 2 set + 1
        const float la = args.level_a, lb = args.level_b;
        const bool protect = args.n_sink > 0 || args.n_recent > 0;
        const int nslot = args.n_sink + args.n_recent;
        const int recent0 = L - args.n_recent;
        const int t = 32 * q + lane, tp = t >> 6, trow = t & 63;     // token of the tile (S lane)
        // softmax of this set's eight heads (hb .. hb + 7): running reference maximum and
        // sum per head; both sets take part, each with its own named barrier
        constexpr int kH = kTmHeads / 2;
        const int hb = kH * set;
        float m_ref[kH], l[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) { m_ref[h] = -INFINITY; l[h] = 0.f; }
        // softmax of tile i: runs after the token-major x of tile i + 1 is written, so it
        // overlaps that tile's QK instead of delaying it
        auto softmax_tile = [&](int i) {
            const int bi = i & 1;
            const int pos = (first_page + 2 * i + (t >> 6)) * kPageTok + (t & 63);
            const bool valid = tm_page_ok(args, b, first_page, T, 2 * i + (t >> 6)) && pos < L;
            mbar_wait(smem_u32(&sm.sfull[bi]), (unsigned)((i >> 1) & 1), &sm.abort);
            __syncwarp();
            tc_fence_after();
            uint32_t u[kH];
            tmem_ld8(tmem + lane_base + kTmColS + kTmHeads * bi + hb, u);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(smem_u32(&sm.sfree[bi]));
            float s[kH];
            bool up = false;
#pragma unroll
            for (int h = 0; h < kH; ++h) {
                s[h] = valid ? __uint_as_float(u[h]) * args.scale_log2 : -INFINITY;
                up |= s[h] > m_ref[h] + kRescaleLog2 || (m_ref[h] == -INFINITY && s[h] > -INFINITY);
            }
            const bool wup = __any_sync(0xffffffffu, up);
            if (lane == 0) sm.vote[set][bi][q] = wup ? 1 : 0;
            named_bar_sync(1 + set, 128);
            const bool any = (sm.vote[set][bi][0] | sm.vote[set][bi][1] | sm.vote[set][bi][2] | sm.vote[set][bi][3]) != 0;
            if (any) {
                // per-head maximum over the tile's 128 tokens
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    float mx = s[h];
#pragma unroll
                    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    if (lane == 0) sm.red[set][q][h] = mx;
                }
                named_bar_sync(1 + set, 128);
                if (q == 0 && lane < kH) {
                    const int h = hb + lane;
                    const float tm = fmaxf(fmaxf(sm.red[set][0][lane], sm.red[set][1][lane]),
                                           fmaxf(sm.red[set][2][lane], sm.red[set][3][lane]));
                    const float mo = sm.mref[h];
                    float al = 1.f, mn = mo;
                    if (tm > mo + kRescaleLog2 || (mo == -INFINITY && tm > -INFINITY)) {
                        al = (mo == -INFINITY) ? 0.f : ex2(mo - tm);
                        mn = tm;
                    }
                    sm.alpha[h] = al;
                    sm.mref[h] = mn;
                }
                named_bar_sync(1 + set, 128);
                bool moved = false;
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    const float al = sm.alpha[hb + h];
                    m_ref[h] = sm.mref[hb + h];
                    l[h] *= al;
                    moved |= al != 1.f;
                }
                if (moved && i > 0) {
                    // O holds PV of tiles 0..i-1: wait for PV(i-1), scale this set's heads in
                    // this quarter's lanes
                    mbar_wait(smem_u32(&sm.pvdone[(i - 1) & 1]), (unsigned)(((i - 1) >> 1) & 1), &sm.abort);
                    __syncwarp();
                    tc_fence_after();
#pragma unroll 1
                    for (int g = 0; g < ROLAQ_GROUPS; ++g) {
                        uint32_t v[kH];
                        tmem_ld8(tmem + lane_base + kTmColO + 16 * g + hb, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < kH; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) * sm.alpha[hb + h]);
                        tmem_st8(tmem + lane_base + kTmColO + 16 * g + hb, v);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                }
                named_bar_sync(1 + set, 128);  // red / alpha are read by every warp of the set before reuse
            }
            // P buffer bi is free once PV(i - 2) has completed
            if (i >= 2) mbar_wait(smem_u32(&sm.pvdone[bi]), (unsigned)(((i - 2) >> 1) & 1), &sm.abort);
            uint32_t pw[kH / 2];
#pragma unroll
            for (int h2 = 0; h2 < kH / 2; ++h2) {
                const float p0 = (m_ref[2 * h2] == -INFINITY) ? 0.f : ex2(s[2 * h2] - m_ref[2 * h2]);
                const float p1 = (m_ref[2 * h2 + 1] == -INFINITY) ? 0.f : ex2(s[2 * h2 + 1] - m_ref[2 * h2 + 1]);
                l[2 * h2] += p0;
                l[2 * h2 + 1] += p1;
                pw[h2] = pack_f16(p0, p1);
            }
            // row t of P: heads 0-7 in 16-byte chunk 0, heads 8-15 in chunk 1 (32-byte swizzle)
            *reinterpret_cast<uint4*>(sm.P[bi] + t * 32 + ((set ^ ((t >> 2) & 1)) << 4)) =
                make_uint4(pw[0], pw[1], pw[2], pw[3]);
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive_lane0(smem_u32(&sm.pready[bi]));
        };
        for (int i = 0; i < nt; ++i) {
            const int st = i % kTmStages;
            mbar_wait(smem_u32(&sm.full[st]), (unsigned)((i / kTmStages) & 1), &sm.abort);
            if (i >= 3) mbar_wait(smem_u32(&sm.tbl_free[i % 3]), (unsigned)((i / 3 - 1) & 1), &sm.abort);
            const int pos = (first_page + 2 * i + tp) * kPageTok + trow;
            const bool valid = tm_page_ok(args, b, first_page, T, 2 * i + tp) && pos < L;
            const bool prot = valid && protect && (pos < args.n_sink || pos >= recent0);
            const __nv_bfloat16* prow = nullptr;
            if (prot) {
                const int slot = pos < args.n_sink ? pos : args.n_sink + pos % args.n_recent;
                prow = args.prot + ((size_t)b * nslot + slot) * ROLAQ_D_C;
            }
            if (i >= 1) mbar_wait(smem_u32(&sm.xq_free[set]), (unsigned)((i - 1) & 1), &sm.abort);
            __syncwarp();
            tc_fence_after();
#pragma unroll 1
            for (int gi = 0; gi < 2; ++gi) {
                const int g = 2 * set + gi;
                uint32_t sc16, mu16;
                tm_token_store(sm.cm[st][tp], trow, g, valid, prot, prow, la, lb,
                               tmem + lane_base + kTmColXq + 64 * g, sc16, mu16);
                uint16_t* te = reinterpret_cast<uint16_t*>(&sm.tbl[i % 3][g][t >> 2]);
                te[t & 3] = (uint16_t)sc16;
                te[4 + (t & 3)] = (uint16_t)mu16;
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_lane0(smem_u32(&sm.xq_full[set]));
            mbar_arrive_lane0(smem_u32(&sm.tbl_full[i % 3]));
            mbar_arrive_lane0(smem_u32(&sm.pfree[st]));
            if (i >= 1) softmax_tile(i - 1);
        }
        if (nt > 0) softmax_tile(nt - 1);
        // ---- this item's partial: O (rows = channel lanes), per-head (m, l), this set's heads
        if (nt > 0) mbar_wait(smem_u32(&sm.pvdone[(nt - 1) & 1]), (unsigned)(((nt - 1) >> 1) & 1), &sm.abort);
        __syncwarp();
        tc_fence_after();
        const int ch_in_group = 32 * q + 4 * (lane & 7) + (lane >> 3);
#pragma unroll 1
        for (int g = 0; g < ROLAQ_GROUPS; ++g) {
            uint32_t v[kH];
            tmem_ld8(tmem + lane_base + kTmColO + 16 * g + hb, v);
            tmem_ld_wait();
            float* dst = args.ws_o + ((size_t)blockIdx.x * args.heads + h0 + hb) * ROLAQ_D_C + 128 * g + ch_in_group;
#pragma unroll
            for (int h = 0; h < kH; ++h) dst[(size_t)h * ROLAQ_D_C] = __uint_as_float(v[h]);
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            float v = l[h];
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) sm.red[set][q][h] = v;
        }
        named_bar_sync(1 + set, 128);
        if (q == 0 && lane < kH) {
            args.ws_ml[(size_t)blockIdx.x * args.heads + h0 + hb + lane] =
                make_float2(sm.mref[hb + lane], (sm.red[set][0][lane] + sm.red[set][1][lane]) +
                                                    (sm.red[set][2][lane] + sm.red[set][3][lane]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmCols) : "memory");
    }
}

}  // namespace rolaq
