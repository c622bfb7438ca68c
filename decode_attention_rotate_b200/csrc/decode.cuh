// Absorbed-MLA decode attention over the packed 2-bit cache ("RoLaQ", §2.1, §3.3):
// scores (q_c_rot . x + q_R . k_R) * sm_scale with x = mean + scale * level(code),
// softmax over the request's tokens, 512-d latent readout in the rotated basis.
//
// Kernel A (rolaq_decode_split<HC>): one CTA per (work item, chunk of HC = 16 or 32 query
// heads).  A work item is a run of whole pages of one request (split-K over the sequence),
// one item per SM in the plan.  Each 64-token page is one tile, handled by warps with
// fixed roles and handed on through mbarriers:
//   warp 0 (lane 0)   streams the pages (one 144-row bulk tensor copy each, 128-byte
//                     swizzle) through kStages shared-memory stages (3, or 2 with
//                     32 heads);
//   warps 8..15       dequantise: thread (token t, group g) forms the four fp16 values
//                     mean + scale * level of its (token, group) and turns its 128 codes
//                     into x with one PRMT per pair (one selector per four codes), then
//                     writes x twice: token-major into tensor memory (M = 64 layout, QK's
//                     A operand) and into a 128-byte-swizzled shared-memory tile
//                     [64 tokens][512 channels] (PV's A operand; two tiles).  fp16, not
//                     bf16: channels sharing a code share one rounding error, which bf16
//                     makes ~5x too large in the output;
//   warp 1            issues QK (warp-uniform loop, one elected lane per batch of
//                     instructions): tcgen05.mma M = 64 tokens, N = HC heads, K = 512
//                     (fp16, A = x in tensor memory) plus K = 64 (bf16, A = the staged
//                     page's RoPE rows), S in tensor memory;
//   warp 2            issues PV: tcgen05.mma M = 128 channels of a group, N = HC heads,
//                     K = 64 tokens, A = the shared-memory tile read transposed
//                     (MN-major), B = P, O (fp32) accumulated in tensor memory;
//   warps 4..7        softmax (softmax_role): one tensor-memory load gives a token's HC
//                     scores; the running max moves only when a score exceeds it by more
//                     than 2^8 (one reducing barrier per page decides), in which case O
//                     is rescaled before the next PV; P goes to shared memory (three
//                     buffers) as the fp16 B operand.
// Every kernel here is launched as a programmatic dependent of the previous one in the
// stream and waits (griddepcontrol.wait) before it reads an input.
// Kernel B (rolaq_decode_merge): log-sum-exp merge of the per-item partials.
//
// Fused append (one new token per request at position L - 1, the per-step write of a
// serving decode): in kernel A the otherwise idle warp 3 of every CTA of head chunk 0
// computes a slice of the new tokens' rotated coordinates y = c . R into the workspace,
// while the item pages exclude position L - 1 (the plan covers L - 1 tokens; the
// protected window still counts L).  Kernel B, which runs after A, completes the append
// for its request (group statistics, codes, the page record and side-store row, written
// by the head-0 CTA) and adds the new token's term to the merge.
#pragma once
#include "common.cuh"

namespace rolaq {

constexpr int kPageTok = ROLAQ_PAGE_TOKENS;
constexpr int kPageRows = ROLAQ_PAGE_BYTES / 128;   // 144 rows of 128 B
constexpr int kDecodeThreads = 512;
// HC = query heads per CTA (16 or 32): the N of both tensor-core products.
template <int HC> __host__ __device__ constexpr int stages_for() { return HC == 16 ? 3 : 2; }   // pages in flight
constexpr int kSoftWarp0 = 4;                       // softmax warps 4..7 (TMEM lane quarters)
constexpr int kDqWarp0 = 8;                         // dequant warps 8..15
constexpr int kXAtom = kPageTok * 128;              // one 64-channel column block of an x tile
constexpr int kXTile = 8 * kXAtom;                  // 64 KB: 64 tokens x 512 fp16
constexpr int kMetaRow = 64;                        // page rows: codes 0..63, meta 64..79,
constexpr int kKrRow = 80;                          // RoPE keys 80..143
constexpr int kSCol = 0;                            // TMEM: S tiles at columns 0 and HC
constexpr int kOCol = 64;                           //       O at 64.. (HC per group)
constexpr int kXqCol = 256;                         //       token-major x (QK's A): 256..511
template <int HC> __host__ __device__ constexpr int tmem_cols_for() { return 512; }
constexpr int kPBufs = 3;                           // probability buffers (PV's B operand)
constexpr float kRescaleLog2 = 8.f;
constexpr float kF16Max = 65504.f;

struct DecodeArgs {
    const int32_t* page_table;
    int64_t num_pages;
    int max_pages;
    const __nv_bfloat16* prot;   // [batch][n_sink + n_recent][512] or null
    int n_sink, n_recent;
    const __nv_bfloat16* q;      // [batch][heads][512]
    const __nv_bfloat16* qr;     // [batch][heads][64]
    const int32_t* seq_lens;
    int batch, heads;
    float scale_log2;            // sm_scale * log2(e)
    float level_a, level_b;      // reconstruction levels (fp32)
    int target_items;
    float* ws_o;                 // [items][heads][512]  sum_t 2^(s_t - m) x_t
    float2* ws_ml;               // [items][heads]       (m (log2 units), sum_t 2^(s_t - m))
    // fused append (append = 1): new token of request b at position seq_lens[b] - 1
    int append;
    const __nv_bfloat16* app_R;  // rotation planes [3][512][512] (row = output coordinate)
    const __nv_bfloat16* app_c;  // new content latents [batch][512]
    float* ws_y;                 // [batch][512] their rotated coordinates
};

// What the merge needs to complete a fused append.  y == nullptr: no append.
struct AppendArgs {
    const float* y;              // [batch][512] rotated coordinates of the new tokens
    const __nv_bfloat16* k_r;    // [batch][64] their RoPE keys
    const __nv_bfloat16* q;      // [batch][heads][512] rotated content queries
    const __nv_bfloat16* qr;     // [batch][heads][64]
    float scale_log2, tau, gain, level_a, level_b;
    uint8_t* pages;
    const int32_t* page_table;
    int64_t num_pages;
    int max_pages;
    __nv_bfloat16* prot;         // [batch][n_sink + n_recent][512] or null
    int n_sink, n_recent;
};

template <int HC>
struct DecodeSmem {
    static constexpr int kStages = stages_for<HC>();
    alignas(1024) uint8_t x[2][kXTile];                   // x tiles (K-major, 128-byte swizzle)
    alignas(1024) uint8_t stage[kStages][ROLAQ_PAGE_BYTES];
    alignas(128) uint8_t qc[HC * ROLAQ_D_C * 2];          // fp16 query, QK B operand
    alignas(128) uint8_t qr[HC * ROLAQ_D_R * 2];          // bf16 RoPE query, B operand
    alignas(128) uint8_t P[kPBufs][HC * kPageTok * 2];    // fp16 probabilities, PV B operand
    float red[4][HC];                                     // softmax warps: per-warp head values
    float mref[HC];                                       // running reference max per head
    float alpha[HC];                                      // its last rescale factor
    alignas(8) uint64_t full[kStages];     // page copy landed
    alignas(8) uint64_t pfree[kStages];    // page read by the dequant warps and the QK MMAs
    alignas(8) uint64_t xready[2][2];      // x tile half written (channel groups 0-1 / 2-3)
    alignas(8) uint64_t xfree[2][2];       // PV of the tile done for groups 0-1 / all groups
    alignas(8) uint64_t xq_full[2];        // token-major x in tensor memory written (groups 0-1 / 2-3)
    alignas(8) uint64_t xq_free;           // QK of the page done with the token-major x
    alignas(8) uint64_t sfull[2];          // QK of the tile done
    alignas(8) uint64_t sfree[2];          // scores read by the softmax warps
    alignas(8) uint64_t pready[kPBufs];    // P written (and O rescaled if needed)
    alignas(8) uint64_t pdone[kPBufs];     // PV done with the P buffer
    int valid[kStages];
    uint32_t tmem_base;
    int plan[4];
    int abort;
};
static_assert(sizeof(DecodeSmem<16>) + 1024 <= 227 * 1024, "decode shared memory (16 heads)");
static_assert(sizeof(DecodeSmem<32>) + 1024 <= 227 * 1024, "decode shared memory (32 heads)");

// ---- split plan --------------------------------------------------------------
// pages_b = ceil(L_b / 64); chunk = the smallest value >= max(1, ceil(sum_b pages_b /
// target)) for which the item count sum_b ceil(pages_b / chunk) is at most `target` (one
// wave of items when `target` is the SM count), or that first value when no chunk fits
// (more requests than `target`); request b gets ceil(pages_b / chunk) items numbered
// consecutively in request order.  Executed by one full warp; every lane returns the same
// values.
struct PlanInfo { int b, first_page, n_pages, n_items, item_offset, chunk; };

// app = 1 (fused append): the items cover L - 1 tokens of a request of length L.
__device__ __forceinline__ int plan_pages(const int32_t* seq_lens, int b, int app) {
    return (max(seq_lens[b] - app, 0) + kPageTok - 1) / kPageTok;
}

__device__ __forceinline__ int plan_items(const int32_t* seq_lens, int batch, int chunk, int app) {
    const int lane = threadIdx.x & 31;
    int items = 0;
    for (int b = lane; b < batch; b += 32) {
        const int pages = plan_pages(seq_lens, b, app);
        items += (pages + chunk - 1) / chunk;
    }
    for (int o = 16; o; o >>= 1) items += __shfl_xor_sync(0xffffffffu, items, o);
    return items;
}

__device__ __forceinline__ int plan_chunk(const int32_t* seq_lens, int batch, int target, int app) {
    const int lane = threadIdx.x & 31;
    long long total = 0;
    int max_pages = 0;
    for (int b = lane; b < batch; b += 32) {
        const int pages = plan_pages(seq_lens, b, app);
        total += pages;
        max_pages = max(max_pages, pages);
    }
    for (int o = 16; o; o >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, o);
        max_pages = max(max_pages, __shfl_xor_sync(0xffffffffu, max_pages, o));
    }
    int c = (int)max(1LL, (total + target - 1) / target);
    // ragged lengths can leave more items than `target` (a second, mostly idle wave);
    // with chunk = max_pages every non-empty request is one item, so when batch <=
    // target a fitting chunk exists: binary search for the smallest
    if (batch <= target && max_pages > c && plan_items(seq_lens, batch, c, app) > target) {
        int lo = c + 1, hi = max_pages;
        while (lo < hi) {
            const int mid = lo + (hi - lo) / 2;
            if (plan_items(seq_lens, batch, mid, app) <= target) hi = mid;
            else lo = mid + 1;
        }
        c = lo;
    }
    return c;
}

// Locate work item `item` (or request `req` when item < 0).  n_items = total item count.
__device__ PlanInfo plan_lookup(const int32_t* seq_lens, int batch, int target, int item,
                                int req, int app) {
    const int lane = threadIdx.x & 31;
    PlanInfo pi{-1, 0, 0, 0, 0, 0};
    const int chunk = plan_chunk(seq_lens, batch, target, app);
    pi.chunk = chunk;
    int base = 0;
    for (int b0 = 0; b0 < batch; b0 += 32) {
        int b = b0 + lane;
        int items = 0, pages = 0;
        if (b < batch) {
            pages = plan_pages(seq_lens, b, app);
            items = (pages + chunk - 1) / chunk;
        }
        int incl = items;
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int excl = base + incl - items;
        bool hit = (b < batch) && ((item >= 0) ? (item >= excl && item < excl + items) : (b == req));
        unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            int src = __ffs(m) - 1;
            int e = __shfl_sync(0xffffffffu, excl, src);
            int it = __shfl_sync(0xffffffffu, items, src);
            int pg = __shfl_sync(0xffffffffu, pages, src);
            pi.b = b0 + src;
            pi.item_offset = e;
            pi.n_items = it;
            if (item >= 0) {
                int j = item - e;
                pi.first_page = j * chunk;
                pi.n_pages = min(chunk, pg - j * chunk);
            } else {
                pi.first_page = 0;
                pi.n_pages = pg;
            }
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (item >= 0 && pi.b < 0) pi.n_items = base;   // item past the end
    return pi;
}

// Sixteen codes of one token (one 32-bit word) into fp16 pairs, one selector per four
// codes: r[k][0] = (x of byte 0's code k, x of byte 1's code k), r[k][1] the same for
// bytes 2 and 3.  The lookup pair (lo, hi) holds the low and high bytes of the token's
// four fp16 values, so selector nibbles (c, c + 4) pick value c; the second pair uses the
// selector's upper half.
__device__ __forceinline__ void codes_to_x(uint32_t w, uint2 lut, uint32_t (&r)[4][2]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t m = (w >> (2 * k)) & 0x03030303u;
        const uint32_t sel = m * 0x11u + 0x40404040u;
        r[k][0] = prmt(lut.x, lut.y, sel);
        r[k][1] = prmt(lut.x, lut.y, sel >> 16);
    }
}

// ---- tensor-core operands -----------------------------------------------------
// Instruction descriptors: fp32 accumulate, K-major unless noted, N = HC heads.
template <int HC> __host__ __device__ constexpr uint32_t id_qk() { return (1u << 4) | ((uint32_t)(HC >> 3) << 17) | ((64u >> 4) << 24); }  // f16, M = 64
template <int HC> __host__ __device__ constexpr uint32_t id_rope() { return id_qk<HC>() | (1u << 7) | (1u << 10); }                      // bf16, M = 64
template <int HC> __host__ __device__ constexpr uint32_t id_pv() {                                                                      // f16, M = 128, A MN-major
    return (1u << 4) | (1u << 15) | ((uint32_t)(HC >> 3) << 17) | ((128u >> 4) << 24);
}

// Column slot of channel order inside every 16-channel block: the PRMT lookup yields the
// pairs (k, k+4), so slot 2k + e of a block of 8 holds channel k + 4e.  The query is laid
// out in slot order and O rows come back in slot order; this maps a slot to its channel.
__host__ __device__ __forceinline__ int slot_channel(int s) {
    return (s & ~7) + ((s & 7) >> 1) + 4 * (s & 1);
}
// Byte offset of (row, 16-byte chunk) in an x tile: 64-channel column blocks of
// [64 rows][128 B], chunks XOR row % 8 (the tensor cores' 128-byte swizzle).
__device__ __forceinline__ uint32_t x_off(int row, int chunk) {
    return (chunk >> 3) * kXAtom + row * 128 + ((((chunk & 7) ^ row) & 7) << 4);
}
// K-major operand without swizzle (8-row x 16-byte core matrices, K-adjacent cores 128 B
// apart, 8-row groups `sbo` apart): byte offset of element (row n, k), 2-byte elements.
__device__ __forceinline__ uint32_t plain_off(int n, int k, int sbo) {
    return (n >> 3) * sbo + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

// Page-table entry of page `page_idx` of request b (-1 past the table).
__device__ __forceinline__ long long page_id(const DecodeArgs& args, int b, int page_idx) {
    return page_idx < args.max_pages ? (long long)args.page_table[(long long)b * args.max_pages + page_idx] : -1;
}
__device__ __forceinline__ bool page_ok(const DecodeArgs& args, long long pid) {
    return pid >= 0 && pid < args.num_pages;
}
// Issue the bulk copy of one page (all 144 rows) into stage k % kStages, or mark the
// stage invalid when the page-table entry is outside the pool.
template <int HC>
__device__ __forceinline__ void load_page(DecodeSmem<HC>& sm, const CUtensorMap* map, const DecodeArgs& args,
                                          long long pid, int k) {
    const int st = k % DecodeSmem<HC>::kStages;
    const uint32_t bar = smem_u32(&sm.full[st]);
    if (page_ok(args, pid)) {
        sm.valid[st] = 1;
        mbar_arrive_expect_tx(bar, ROLAQ_PAGE_BYTES);
        tma_load_2d(smem_u32(sm.stage[st]), map, 0, (int)(pid * kPageRows), bar);
    } else {
        sm.valid[st] = 0;
        raise_status(ROLAQ_STATUS_BAD_PAGE);
        mbar_arrive(bar);
    }
}

// One dequant thread's share of a tile: token row t, channel group g.  The four fp16
// values mean + scale * (-b, -a, a, b) are split into low and high bytes so that a PRMT
// picks value c with nibbles c and c + 4; each 32-bit word of codes (16 channels) gives
// eight fp16 pairs (o[w][0..3] and o[w][4..7]: two 16-byte chunks of the x tile in slot
// order).  Tokens past the sequence end (or on an invalid page) get x = 0; protected
// tokens take their bf16 side-store row instead of the codes.  Computed into registers
// before the x buffer is free, stored after.
__device__ __forceinline__ void dequant_tile_part(const uint8_t* pg, int t, int g, bool valid, bool prot,
                                                  const __nv_bfloat16* prow, float la, float lb,
                                                  uint32_t (&o)[8][8]) {
    uint2 lut = make_uint2(0u, 0u);
    uint4 cw0 = make_uint4(0u, 0u, 0u, 0u), cw1 = cw0;
    if (valid) {
        const float2 ms = *reinterpret_cast<const float2*>(pg + swz128(kMetaRow + (t >> 2), (t & 3) * 32 + 8 * g));
        if (!(fabsf(ms.x) + fabsf(ms.y) * lb < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        const uint32_t w01 = pack_f16(fmaf(ms.y, -lb, ms.x), fmaf(ms.y, -la, ms.x));
        const uint32_t w23 = pack_f16(fmaf(ms.y, la, ms.x), fmaf(ms.y, lb, ms.x));
        lut.x = prmt(w01, w23, 0x6420u);
        lut.y = prmt(w01, w23, 0x7531u);
        cw0 = *reinterpret_cast<const uint4*>(pg + t * 128 + (((2 * g) ^ (t & 7)) << 4));
        cw1 = *reinterpret_cast<const uint4*>(pg + t * 128 + (((2 * g + 1) ^ (t & 7)) << 4));
    }
    const uint32_t cw[8] = {cw0.x, cw0.y, cw0.z, cw0.w, cw1.x, cw1.y, cw1.z, cw1.w};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        uint32_t r[4][2];
        codes_to_x(cw[w], lut, r);
#pragma unroll
        for (int k = 0; k < 4; ++k) { o[w][k] = r[k][0]; o[w][4 + k] = r[k][1]; }
    }
    if (prot) {
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            // channels 128g + 16w + {0..15} from the side store, in slot order
            const uint4 u0 = reinterpret_cast<const uint4*>(prow + 128 * g + 16 * w)[0];
            const uint4 u1 = reinterpret_cast<const uint4*>(prow + 128 * g + 16 * w)[1];
            const uint32_t v[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                // slot pair k of each 8-block: channels (k, k + 4) of the block
                const float a0 = (k & 1) ? bf16_hi(v[k >> 1]) : bf16_lo(v[k >> 1]);
                const float a1 = (k & 1) ? bf16_hi(v[2 + (k >> 1)]) : bf16_lo(v[2 + (k >> 1)]);
                const float b0 = (k & 1) ? bf16_hi(v[4 + (k >> 1)]) : bf16_lo(v[4 + (k >> 1)]);
                const float b1 = (k & 1) ? bf16_hi(v[6 + (k >> 1)]) : bf16_lo(v[6 + (k >> 1)]);
                o[w][k] = pack_f16(a0, a1);
                o[w][4 + k] = pack_f16(b0, b1);
            }
        }
    }
}
__device__ __forceinline__ void store_tile_part(uint8_t* xt, int t, int g, const uint32_t (&o)[8][8]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int chunk = 16 * g + 2 * w;          // 16-byte chunk index along the 512 slots
        *reinterpret_cast<uint4*>(xt + x_off(t, chunk)) = make_uint4(o[w][0], o[w][1], o[w][2], o[w][3]);
        *reinterpret_cast<uint4*>(xt + x_off(t, chunk + 1)) = make_uint4(o[w][4], o[w][5], o[w][6], o[w][7]);
    }
}

// Scores of one softmax warp: 16 TMEM lanes x HC columns (16x256b shape, HC / 8 repeats).
__device__ __forceinline__ void tmem_ld_scores(uint32_t taddr, uint32_t (&u)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_scores(uint32_t taddr, uint32_t (&u)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x4.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
                   "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
                   "=r"(u[15])
                 : "r"(taddr));
}

// Fused append, kernel A part (one warp): output coordinates o = cta, cta + ncta, ... of
// every new token, y[b][o] = sum_k c[b][k] R[k][o].  Lane l takes inputs 16l .. 16l + 15:
// the three rotation planes summed in fp32 (smallest first), fma with the latents, then a
// butterfly over the warp.
__device__ __forceinline__ void append_rotate(const DecodeArgs& args, int cta, int ncta) {
    const int lane = threadIdx.x & 31;
    const size_t plane = (size_t)ROLAQ_D_C * ROLAQ_D_C;
    for (int o = cta; o < ROLAQ_D_C; o += ncta) {
        float rk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) rk[i] = 0.f;
#pragma unroll
        for (int pl = 2; pl >= 0; --pl) {
            const uint4* row = reinterpret_cast<const uint4*>(args.app_R + pl * plane + (size_t)o * ROLAQ_D_C);
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                const uint4 u = row[2 * lane + hv];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    rk[8 * hv + 2 * q] += __uint_as_float(w[q] << 16);
                    rk[8 * hv + 2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
                }
            }
        }
        for (int b = 0; b < args.batch; ++b) {
            if (args.seq_lens[b] < 1) continue;
            const uint4* crow = reinterpret_cast<const uint4*>(args.app_c + (size_t)b * ROLAQ_D_C);
            float acc = 0.f;
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                const uint4 cu = crow[2 * lane + hv];
                const uint32_t cw[4] = {cu.x, cu.y, cu.z, cu.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc = fmaf(__uint_as_float(cw[q] << 16), rk[8 * hv + 2 * q], acc);
                    acc = fmaf(__uint_as_float(cw[q] & 0xFFFF0000u), rk[8 * hv + 2 * q + 1], acc);
                }
            }
            for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) args.ws_y[(size_t)b * ROLAQ_D_C + o] = acc;
        }
    }
}

// Softmax role (warps 4..7) of the decode kernels: scores from tensor memory, the lazy
// reference max, P into shared memory (fp16, or bf16 when the x operand is bf16), O
// rescaled in place when the reference moves, and at the end the item's partial (O rows
// in slot order for the 2-bit kernel, in channel order for the bf16 one, and (m, l) per
// head).  pv_wait(j) returns once the PV of page j has completed.
template <bool kBf16P> __device__ __forceinline__ uint16_t p_bits(float p);
template <> __device__ __forceinline__ uint16_t p_bits<false>(float p) { return __half_as_ushort(__float2half_rn(p)); }
template <> __device__ __forceinline__ uint16_t p_bits<true>(float p) { return __bfloat16_as_ushort(__float2bfloat16_rn(p)); }

template <int HC, bool kBf16P, bool kSlotOrder, typename Smem, typename PvWait>
__device__ __forceinline__ void softmax_role(Smem& sm, const DecodeArgs& args, uint32_t tmem, int warp, int lane,
                                             int b, int first_page, int T, int Lkv, int h0, PvWait pv_wait) {
    // ------------------------------------------------------------- softmax ----
    // Warp q reads TMEM lane quarter q: S rows 16q..16q+15 (M = 64) in lanes 0..15 with
    // the 16x256b shape, so lane (r, i) holds rows 16q + r and 16q + r + 8 of heads
    // 8k + 2i and 8k + 2i + 1 (k < HC / 8); O rows (slots) 32q..32q+31 of every group.
    constexpr int kE = HC / 4;             // heads per thread
    const int q = warp - kSoftWarp0;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int r = lane >> 2, i4 = lane & 3;
    const int rows[2] = {16 * q + r, 16 * q + r + 8};
    int heads[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) heads[e] = 8 * (e >> 1) + 2 * i4 + (e & 1);
    float m_ref[kE], l[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) { m_ref[e] = -INFINITY; l[e] = 0.f; }
    long long pid_next = page_id(args, b, first_page);
    for (int i = 0; i < T; ++i) {
        const int bi = i & 1;
        const bool vpage = page_ok(args, pid_next);
        if (i + 1 < T) pid_next = page_id(args, b, first_page + i + 1);
        mbar_wait(smem_u32(&sm.sfull[bi]), (unsigned)((i >> 1) & 1), &sm.abort);
        __syncwarp();
        tc_fence_after();
        uint32_t u[HC / 2];
        tmem_ld_scores(tmem + lane_base + kSCol + HC * bi, u);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.sfree[bi]));
        // s[e][j]: head heads[e], row rows[j]
        float s2[kE][2];
        bool up = false;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const bool valid = vpage && (first_page + i) * kPageTok + rows[j] < Lkv;
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                const uint32_t raw = u[(e >> 1) * 4 + 2 * j + (e & 1)];
                s2[e][j] = valid ? __uint_as_float(raw) * args.scale_log2 : -INFINITY;
                up |= s2[e][j] > m_ref[e] + kRescaleLog2 || (m_ref[e] == -INFINITY && s2[e][j] > -INFINITY);
            }
        }
        // the four softmax warps agree on whether any head's reference moves
        const bool any = named_bar_or(1, 128, up);
        if (any) {
            // per-head max over the tile: lanes sharing i4 hold the same heads
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                float mx = fmaxf(s2[e][0], s2[e][1]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                if (r == 0) sm.red[q][heads[e]] = mx;
            }
            named_bar_sync(1, 128);
            if (q == 0 && lane < HC) {
                // one thread per head: new reference and factor for all warps
                const int h = lane;
                const float tm = fmaxf(fmaxf(sm.red[0][h], sm.red[1][h]), fmaxf(sm.red[2][h], sm.red[3][h]));
                const float mo = sm.mref[h];
                float al = 1.f, mn = mo;
                if (tm > mo + kRescaleLog2 || (mo == -INFINITY && tm > -INFINITY)) {
                    al = (mo == -INFINITY) ? 0.f : ex2(mo - tm);
                    mn = tm;
                }
                sm.alpha[h] = al;
                sm.mref[h] = mn;
            }
            named_bar_sync(1, 128);
            bool moved = false;
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                const float al = sm.alpha[heads[e]];
                m_ref[e] = sm.mref[heads[e]];
                l[e] *= al;
            }
#pragma unroll
            for (int h = 0; h < HC; ++h) moved |= sm.alpha[h] != 1.f;
            if (moved && i > 0) {
                // O holds PV of tiles 0..i-1: wait for PV(i-1), scale this quarter's lanes
                pv_wait(i - 1);
                __syncwarp();
                tc_fence_after();
#pragma unroll 1
                for (int gc = 0; gc < 4 * (HC / 16); ++gc) {       // 16-column slices of O
                    uint32_t v[16];
                    tmem_ld16(tmem + lane_base + kOCol + 16 * gc, v);
                    tmem_ld_wait();
                    const int hb = 16 * (gc % (HC / 16));            // first head of the slice
#pragma unroll
                    for (int h = 0; h < 16; ++h) v[h] = __float_as_uint(__uint_as_float(v[h]) * sm.alpha[hb + h]);
                    tmem_st16(tmem + lane_base + kOCol + 16 * gc, v);
                }
                tmem_st_wait();
                tc_fence_before();
            }
            named_bar_sync(1, 128);        // red / alpha are read by every softmax warp before reuse
        }
        // P buffer i % kPBufs is free once PV(i - kPBufs) has completed
        const int pi = i % kPBufs;
        if (i >= kPBufs) mbar_wait(smem_u32(&sm.pdone[pi]), (unsigned)((i / kPBufs - 1) & 1), &sm.abort);
        uint8_t* P = sm.P[pi];
#pragma unroll
        for (int e = 0; e < kE; ++e)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float p = (m_ref[e] == -INFINITY) ? 0.f : ex2(s2[e][j] - m_ref[e]);
                l[e] += p;
                *reinterpret_cast<uint16_t*>(P + plain_off(heads[e], rows[j], 8 * 128)) = p_bits<kBf16P>(p);
            }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.pready[pi]));
    }
    // ---- this item's partial: O (rows = slots), per-head (m, l) ----------------
    if (T > 0) pv_wait(T - 1);
    __syncwarp();
    tc_fence_after();
    const int m = 32 * q + lane;           // O row = slot (or channel) within the group
#pragma unroll 1
    for (int gc = 0; gc < 4 * (HC / 16); ++gc) {           // 16-column slices of O
        const int g = gc / (HC / 16), hb = 16 * (gc % (HC / 16));
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + kOCol + 16 * gc, v);
        tmem_ld_wait();
        float* dst = args.ws_o + ((size_t)blockIdx.x * args.heads + h0 + hb) * ROLAQ_D_C + 128 * g + (kSlotOrder ? slot_channel(m) : m);
#pragma unroll
        for (int h = 0; h < 16; ++h) dst[(size_t)h * ROLAQ_D_C] = __uint_as_float(v[h]);
    }
    // row sums: lanes sharing i4 (8 per warp) and the four warps
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        float v = l[e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        if (r == 0) sm.red[q][heads[e]] = v;
    }
    named_bar_sync(1, 128);
    if (q == 0 && lane < HC) {
        const int h = lane;
        args.ws_ml[(size_t)blockIdx.x * args.heads + h0 + h] =
            make_float2(sm.mref[h], (sm.red[0][h] + sm.red[1][h]) + (sm.red[2][h] + sm.red[3][h]));
    }
}

template <int HC>
__global__ void __launch_bounds__(kDecodeThreads, 1)
rolaq_decode_split(const __grid_constant__ CUtensorMap map_page, const DecodeArgs args) {
    extern __shared__ uint8_t smem_raw[];
    constexpr int kStages = DecodeSmem<HC>::kStages;
    constexpr int kTmemCols = tmem_cols_for<HC>();
    constexpr uint32_t kIdQk = id_qk<HC>(), kIdRope = id_rope<HC>(), kIdPv = id_pv<HC>();
    // offset the __shared__ array itself (not an integer address) so that every access
    // stays a shared-memory access
    DecodeSmem<HC>& sm =
        *reinterpret_cast<DecodeSmem<HC>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hc = blockIdx.y;                 // HC-head chunk
    // launched as a programmatic dependent of the previous kernel in the stream: wait for
    // it before the first read of any input or write of the workspace
    grid_dependency_wait();

    if (warp == 0) {
        PlanInfo pi = plan_lookup(args.seq_lens, args.batch, args.target_items, (int)blockIdx.x, -1, args.append);
        if (lane == 0) {
            sm.plan[0] = pi.b;
            sm.plan[1] = pi.first_page;
            sm.plan[2] = pi.n_pages;
        }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.pfree[s]), (kDecodeThreads / 32 - kDqWarp0) + 1);
        }
        for (int s = 0; s < 2; ++s) {
            for (int hf = 0; hf < 2; ++hf) {
                mbar_init(smem_u32(&sm.xready[s][hf]), (kDecodeThreads / 32 - kDqWarp0) / 2);
                mbar_init(smem_u32(&sm.xfree[s][hf]), 1);
            }
            mbar_init(smem_u32(&sm.sfull[s]), 1);
            mbar_init(smem_u32(&sm.sfree[s]), 4);
        }
        for (int s = 0; s < kPBufs; ++s) {
            mbar_init(smem_u32(&sm.pready[s]), 4);
            mbar_init(smem_u32(&sm.pdone[s]), 1);
        }
        for (int hf = 0; hf < 2; ++hf) mbar_init(smem_u32(&sm.xq_full[hf]), (kDecodeThreads / 32 - kDqWarp0) / 2);
        mbar_init(smem_u32(&sm.xq_free), 1);
        for (int h = 0; h < HC; ++h) sm.mref[h] = -INFINITY;
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_page);
    }
    __syncthreads();
    const int b = sm.plan[0];
    const bool appender = args.append && blockIdx.y == 0 && warp == 3;
    if (b < 0) {                               // item past the end of the plan
        if (appender) append_rotate(args, (int)blockIdx.x, (int)gridDim.x);
        return;
    }
    const int first_page = sm.plan[1], T = sm.plan[2];
    const int L = args.seq_lens[b];            // protected window: the last n_recent of L
    const int Lkv = L - args.append;           // tokens read from the pages
    const int h0 = hc * HC;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // queries as B operands: fp16 content query in slot order, bf16 RoPE query
    {
        const uint16_t* qb = reinterpret_cast<const uint16_t*>(args.q + ((size_t)b * args.heads + h0) * ROLAQ_D_C);
        float qmax = 0.f;
        for (int e = threadIdx.x; e < HC * ROLAQ_D_C / 2; e += kDecodeThreads) {
            const int n = e / (ROLAQ_D_C / 2), s = 2 * (e % (ROLAQ_D_C / 2));
            const float v0 = __uint_as_float((uint32_t)qb[n * ROLAQ_D_C + slot_channel(s)] << 16);
            const float v1 = __uint_as_float((uint32_t)qb[n * ROLAQ_D_C + slot_channel(s + 1)] << 16);
            qmax = fmaxf(qmax, fmaxf(fabsf(v0), fabsf(v1)));
            *reinterpret_cast<uint32_t*>(sm.qc + plain_off(n, s, 64 * 128)) = pack_f16(v0, v1);
        }
        if (!(qmax < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        const uint32_t* rb = reinterpret_cast<const uint32_t*>(args.qr + ((size_t)b * args.heads + h0) * ROLAQ_D_R);
        for (int e = threadIdx.x; e < HC * ROLAQ_D_R / 2; e += kDecodeThreads) {
            const int n = e / (ROLAQ_D_R / 2), k = 2 * (e % (ROLAQ_D_R / 2));
            *reinterpret_cast<uint32_t*>(sm.qr + plain_off(n, k, 8 * 128)) = rb[e];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    auto page_of = [&](int k) { return first_page + k; };
    if (threadIdx.x == 0) grid_launch_dependents();     // the merge may be scheduled as CTAs finish

    if (warp == 0) {
        // ------------------------------------------------------------ producer ----
        if (lane == 0)
            for (int k = 0; k < T; ++k) {
                const int st = k % kStages;
                if (k >= kStages)
                    mbar_wait(smem_u32(&sm.pfree[st]), (unsigned)((k / kStages - 1) & 1), &sm.abort);
                load_page(sm, &map_page, args, page_id(args, b, page_of(k)), k);
            }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- QK issue ----
        // The whole warp runs this loop (warp-uniform descriptors); each MMA and commit is
        // issued by one elected lane.
        {
            // Descriptors are built once; an MMA adds a compile-time byte offset / 16 to the
            // start-address field (shared addresses stay below 256 KB, so it never carries).
            const uint64_t dqc = smem_desc(smem_u32(sm.qc), 128, 64 * 128, 0);
            const uint64_t dqr = smem_desc(smem_u32(sm.qr), 128, 8 * 128, 0);
            // (buffers of one kind are contiguous: buffer n starts n * size bytes later)
            const uint64_t dkr = smem_desc(smem_u32(sm.stage[0]) + kKrRow * 128, 16, 1024, 2);
            for (int i = 0; i < T; ++i) {
                const int bi = i & 1, st = i % kStages;
                if (i >= 2) mbar_wait(smem_u32(&sm.sfree[bi]), (unsigned)(((i - 2) >> 1) & 1), &sm.abort);
                const uint64_t dk = dkr + (uint64_t)(st * (ROLAQ_PAGE_BYTES >> 4));
                const uint32_t d = tmem + kSCol + HC * bi;
                // QK from the token-major x in tensor memory (M = 64: token r in lane
                // 32 (r / 16) + r % 16), channel groups 0-1 (K steps 0..15) as soon as that
                // half is written, then groups 2-3 and the RoPE keys
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    mbar_wait(smem_u32(&sm.xq_full[hf]), (unsigned)(i & 1), &sm.abort);
                    __syncwarp();
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int k2 = 0; k2 < ROLAQ_D_C / 32; ++k2) {
                            const int kk = hf * (ROLAQ_D_C / 32) + k2;
                            umma_ts1(d, tmem + kXqCol + 8 * kk, dqc + (uint64_t)((kk * 256) >> 4), kIdQk,
                                     kk > 0 ? 1u : 0u);
                        }
                        if (hf == 1) {
#pragma unroll
                            for (int kk = 0; kk < ROLAQ_D_R / 16; ++kk)
                                umma_ss1(d, dk + (uint64_t)((kk * 32) >> 4), dqr + (uint64_t)((kk * 256) >> 4),
                                         kIdRope, 1u);
                            umma_commit(smem_u32(&sm.sfull[bi]));
                            umma_commit(smem_u32(&sm.pfree[st]));
                            umma_commit(smem_u32(&sm.xq_free));
                        }
                    }
                    __syncwarp();
                }
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------- PV issue ----
        // PV has its own warp, so the PV of page i - 1 never waits behind the QK of page i
        // (different accumulators and operands; each issuing thread's commits track only its
        // own products).
        {
            // x tiles read MN-major (buffers of one kind are contiguous)
            const uint64_t dxm = smem_desc(smem_u32(sm.x[0]), kXAtom, 1024, 2);
            const uint64_t dp = smem_desc(smem_u32(sm.P[0]), 128, 1024, 0);
            auto pv = [&](int j) {
                const int bj = j & 1, pj = j % kPBufs;
                mbar_wait(smem_u32(&sm.pready[pj]), (unsigned)((j / kPBufs) & 1), &sm.abort);
                mbar_wait(smem_u32(&sm.xready[bj][0]), (unsigned)((j >> 1) & 1), &sm.abort);
                mbar_wait(smem_u32(&sm.xready[bj][1]), (unsigned)((j >> 1) & 1), &sm.abort);
                __syncwarp();
                tc_fence_after();
                const uint64_t da = dxm + (uint64_t)(bj * (kXTile >> 4)), db = dp + (uint64_t)(pj * (sizeof(sm.P[0]) >> 4));
                const uint32_t first = j > 0 ? 1u : 0u;
                if (elect_one()) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
#pragma unroll
                        for (int ks = 0; ks < kPageTok / 16; ++ks)
                            umma_ss1(tmem + kOCol + HC * g, da + (uint64_t)((2 * g * kXAtom + ks * 2048) >> 4),
                                     db + (uint64_t)((ks * 256) >> 4), kIdPv, ks > 0 ? 1u : first);
                        if (g == 1) umma_commit(smem_u32(&sm.xfree[bj][0]));   // groups 0-1 read
                    }
                    umma_commit(smem_u32(&sm.xfree[bj][1]));
                    umma_commit(smem_u32(&sm.pdone[pj]));
                }
                __syncwarp();
            };
            for (int j = 0; j < T; ++j) pv(j);
        }
    } else if (warp >= kDqWarp0) {
        // ------------------------------------------------------------- dequant ----
        // warps 8..11 take channel groups 0-1, warps 12..15 groups 2-3
        const int wq = warp - kDqWarp0, hf = wq >> 2;
        const int t = 16 * (wq & 3) + (lane & 15), g = 2 * hf + (lane >> 4);
        const uint32_t xq_lane = (uint32_t)(32 * (warp & 3)) << 16;      // this warp's lane quarter
        const bool protect = args.n_sink > 0 || args.n_recent > 0;
        const int nslot = args.n_sink + args.n_recent;
        const float la = args.level_a, lb = args.level_b;
        for (int i = 0; i < T; ++i) {
            const int bi = i & 1, st = i % kStages;
            mbar_wait(smem_u32(&sm.full[st]), (unsigned)((i / kStages) & 1), &sm.abort);
            const int pos = page_of(i) * kPageTok + t;
            const bool valid = sm.valid[st] && pos < Lkv;
            const bool prot = valid && protect && (pos < args.n_sink || pos >= L - args.n_recent);
            const __nv_bfloat16* prow = nullptr;
            if (prot) {
                const int slot = pos < args.n_sink ? pos : args.n_sink + pos % args.n_recent;
                prow = args.prot + ((size_t)b * nslot + slot) * ROLAQ_D_C;
            }
            uint32_t o[8][8];
            dequant_tile_part(sm.stage[st], t, g, valid, prot, prow, la, lb, o);
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.pfree[st]));      // this warp is done with the page
            // token-major x for QK: lanes 0-15 of this warp's quarter are the tokens, threads
            // 0-15 write group 2 hf and threads 16-31 group 2 hf + 1 (64 columns further)
            if (i >= 1) mbar_wait(smem_u32(&sm.xq_free), (unsigned)((i - 1) & 1), &sm.abort);
            __syncwarp();
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[16];
#pragma unroll
                for (int j = 0; j < 8; ++j) { v[j] = o[2 * c][j]; v[8 + j] = o[2 * c + 1][j]; }
                tmem_st16x32bx2_64(tmem + xq_lane + kXqCol + 128 * hf + 16 * c, v);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.xq_full[hf]));
            // the shared-memory copy (PV's A operand, read MN-major)
            if (i >= 2) mbar_wait(smem_u32(&sm.xfree[bi][hf]), (unsigned)(((i - 2) >> 1) & 1), &sm.abort);
            store_tile_part(sm.x[bi], t, g, o);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.xready[bi][hf]));
        }
    } else if (warp == 3) {
        // --------------------------------------------------------- fused append ----
        if (appender) append_rotate(args, (int)blockIdx.x, (int)gridDim.x);
    } else if (warp >= kSoftWarp0) {
        // ------------------------------------------------------------- softmax ----
        softmax_role<HC, false, true>(sm, args, tmem, warp, lane, b, first_page, T, Lkv, h0, [&](int j) {
            mbar_wait(smem_u32(&sm.xfree[j & 1][1]), (unsigned)((j >> 1) & 1), &sm.abort);
        });
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---- merge --------------------------------------------------------------------
// grid (batch, heads), 512 threads: out[b,h,:] = sum_i w_i o_i / sum_i w_i l_i with
// w_i = 2^(m_i - max m); lse = (max m + log2(sum w l)) * ln 2.  Warp w takes partials
// w, w + 16, ...; lane l owns channels 4l + 128j (j = 0..3), so every thread keeps many
// independent loads in flight; the 16 warp sums are added through shared memory.
// With a fused append, thread c first finishes channel c of request b's new token:
// group statistics over the 128 threads of its group (two-pass mean and population std,
// each a butterfly then the sum of the four warp values), its code, its value x (the
// bf16 y when the new token is protected, else the fp16 mean + scale * level the decode
// reads), and the token's score; the head-0 CTA also stores the token's record.  The new
// token enters the merge as one more partial with m = its score, l = 1, o = x.
constexpr int kMergeThreads = 512;
static_assert(kMergeThreads == ROLAQ_D_C, "merge: one thread per latent channel");

__device__ __forceinline__ float merge_group_sum(float v, float (*red)[4], int g, int gw) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[g][gw] = v;
    __syncthreads();
    const float r = (red[g][0] + red[g][1]) + (red[g][2] + red[g][3]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ float merge_block_sum(float v, float* red) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeThreads / 32; ++w) r += red[w];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kMergeThreads)
rolaq_decode_merge(const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
                   const int32_t* seq_lens, int batch, int heads, int target,
                   float* __restrict__ out, float* __restrict__ lse, const AppendArgs app) {
    __shared__ int s_plan[2];
    __shared__ float s_red[kMergeThreads / 32];
    __shared__ float s_gred[ROLAQ_GROUPS][4];
    __shared__ uint32_t s_codes[ROLAQ_CODE_BYTES / 4];
    __shared__ float s_M, s_den;
    __shared__ __align__(16) float s_acc[kMergeThreads / 32][ROLAQ_D_C];
    const int b = blockIdx.x, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kWarps = kMergeThreads / 32;
    // launched as a programmatic dependent of the split kernel: everything below reads
    // its output, so wait for it (a no-op for an ordinary launch); the next kernel may then
    // be scheduled as merge CTAs finish
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    const int c = threadIdx.x;               // one channel per thread
    if (warp == 0) {
        PlanInfo pi = plan_lookup(seq_lens, batch, target, -1, b, app.y != nullptr ? 1 : 0);
        if (lane == 0) { s_plan[0] = pi.item_offset; s_plan[1] = pi.n_items; }
    }
    // ---- the new token (fused append) ----
    float s_new = -INFINITY, x_new = 0.f;
    const int L = seq_lens[b];
    if (app.y != nullptr && L >= 1) {
        const int g = c >> 7, gw = warp & 3;
        const float y = app.y[(size_t)b * ROLAQ_D_C + c];
        const float mean = merge_group_sum(y, s_gred, g, gw) * (1.f / 128.f);
        const float d = y - mean;
        const float sd = sqrtf(merge_group_sum(d * d, s_gred, g, gw) * (1.f / 128.f));
        const float inv = sd > 0.f ? 1.f / sd : 0.f;
        const float z = d * inv;
        const uint32_t code = (uint32_t)(z >= -app.tau) + (uint32_t)(z >= 0.f) + (uint32_t)(z >= app.tau);
        const float scale = app.gain * sd;
        const int pos = L - 1;
        const bool prot = app.prot != nullptr && (pos < app.n_sink || app.n_recent > 0);
        const float yb = __bfloat162float(__float2bfloat16_rn(y));
        if (prot) {
            x_new = __half2float(__float2half_rn(yb));
        } else {
            const float lev = code == 0 ? -app.level_b : code == 1 ? -app.level_a : code == 2 ? app.level_a : app.level_b;
            x_new = __half2float(__float2half_rn(fmaf(scale, lev, mean)));
            if ((c & 127) == 0 && !(fabsf(mean) + fabsf(scale) * app.level_b < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        }
        const __nv_bfloat16* qb = app.q + ((size_t)b * heads + h) * ROLAQ_D_C;
        float sp = __bfloat162float(qb[c]) * x_new;
        if (c < ROLAQ_D_R)
            sp = fmaf(__bfloat162float(app.qr[((size_t)b * heads + h) * ROLAQ_D_R + c]),
                      __bfloat162float(app.k_r[(size_t)b * ROLAQ_D_R + c]), sp);
        s_new = merge_block_sum(sp, s_red) * app.scale_log2;
        if (h == 0) {
            // the token's record, as the write path stores it
            if (c < ROLAQ_CODE_BYTES / 4) s_codes[c] = 0u;
            __syncthreads();
            atomicOr(&s_codes[c >> 4], code << (2 * (c & 15)));
            __syncthreads();
            long long pid = -1;
            if (pos / ROLAQ_PAGE_TOKENS < app.max_pages) {
                pid = app.page_table[(long long)b * app.max_pages + pos / ROLAQ_PAGE_TOKENS];
                if (pid >= app.num_pages) pid = -1;
            }
            if (pid < 0) {
                if (c == 0) raise_status(ROLAQ_STATUS_BAD_SLOT);
            } else {
                uint8_t* page = app.pages + pid * (long long)ROLAQ_PAGE_BYTES;
                const int row = pos % ROLAQ_PAGE_TOKENS;
                if (c < ROLAQ_CODE_BYTES / 4)
                    reinterpret_cast<uint32_t*>(page + ROLAQ_PAGE_CODES_OFFSET + row * ROLAQ_CODE_BYTES)[c] = s_codes[c];
                if ((c & 127) == 0)
                    *reinterpret_cast<float2*>(page + ROLAQ_PAGE_META_OFFSET + row * ROLAQ_META_BYTES + 8 * g) =
                        make_float2(mean, scale);
                if (c < ROLAQ_KR_BYTES / 8)
                    reinterpret_cast<uint2*>(page + ROLAQ_PAGE_KR_OFFSET + row * ROLAQ_KR_BYTES)[c] =
                        reinterpret_cast<const uint2*>(app.k_r + (size_t)b * ROLAQ_D_R)[c];
                if (prot) {
                    const int nslot = app.n_sink + app.n_recent;
                    const int slot = pos < app.n_sink ? pos : app.n_sink + pos % app.n_recent;
                    app.prot[((size_t)b * nslot + slot) * ROLAQ_D_C + c] = __float2bfloat16_rn(y);
                }
            }
        }
    }
    __syncthreads();
    const int p0 = s_plan[0], np = s_plan[1];
    // max over partials
    float M = -INFINITY;
    for (int p = threadIdx.x; p < np; p += kMergeThreads) M = fmaxf(M, ws_ml[(size_t)(p0 + p) * heads + h].x);
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) s_red[warp] = M;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = s_new;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, s_red[w]);
        s_M = m;
    }
    __syncthreads();
    M = s_M;
    // weighted sums: warp-strided partials, four float4 channel slices per lane
    float4 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M != -INFINITY) {
#pragma unroll 2
        for (int p = warp; p < np; p += kWarps) {
            const float2 ml = ws_ml[(size_t)(p0 + p) * heads + h];
            const float w = ml.y > 0.f ? exp2f(ml.x - M) : 0.f;
            den += w * ml.y;
            const float4* src = reinterpret_cast<const float4*>(ws_o + ((size_t)(p0 + p) * heads + h) * ROLAQ_D_C);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 v = src[lane + 32 * j];
                acc[j].x += w * v.x; acc[j].y += w * v.y; acc[j].z += w * v.z; acc[j].w += w * v.w;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) reinterpret_cast<float4*>(s_acc[warp])[lane + 32 * j] = acc[j];
    if (lane == 0) s_red[warp] = den;
    __syncthreads();
    const float w_new = s_new > -INFINITY ? exp2f(s_new - M) : 0.f;
    if (threadIdx.x == 0) {
        float dsum = 0.f;
        for (int w = 0; w < kWarps; ++w) dsum += s_red[w];
        s_den = dsum + w_new;
    }
    __syncthreads();
    den = s_den;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += s_acc[w][c];
    v = fmaf(w_new, x_new, v);
    out[((size_t)b * heads + h) * ROLAQ_D_C + c] = den > 0.f ? v / den : 0.f;
    if (lse && threadIdx.x == 0)
        lse[(size_t)b * heads + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace rolaq
