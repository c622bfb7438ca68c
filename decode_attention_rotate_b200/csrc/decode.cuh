// Absorbed-MLA decode attention over the packed 2-bit cache ("RoLaQ", §2.1, §3.3):
// scores (q_c_rot . x + q_R . k_R) * sm_scale with x = mean + scale * level(code),
// softmax over the request's tokens, 512-d latent readout in the rotated basis.
//
// Kernel A (rolaq_decode_split): one CTA per (work item, 16-head chunk).  A work item is a
// run of whole pages of one request (split-K over the sequence).  16 warps in four teams
// of four; team t takes pages t, t+4, t+8, ... of the item and keeps its own online
// softmax state, and the four teams are merged inside the CTA at the end, so each item
// writes one partial.  Lane 0 of a team's first warp streams its pages (one 144-row bulk
// tensor copy per page, 128-byte swizzle) through two shared-memory stages and issues the
// team's tensor-core MMAs.  Inside a team, warp q owns content channels 32q..32q+31 of
// every 128-channel group (the TMEM lane quarter it may access) and RoPE channels
// 16q..16q+15.
//
// A team walks its tokens in steps of 16 with one team barrier per step:
//   dequant  per (token, group) the four fp16 values mean + scale * level are prepared
//            one step ahead; a PRMT lookup turns every 2-bit code straight into x (fp16;
//            bf16 would round all channels sharing a code the same way and cost ~5x in
//            output error).
//   QK       mma.sync m16n8k16 (heads = M) on those x fragments in registers; partial
//            scores of the four warps meet in shared memory.
//   A tile   the same fragments transposed (movmatrix) and stored to tensor memory with
//            lanes = channels, columns = tokens (two-slot ring).
//   softmax  warp q takes heads 4q..4q+3; the running max moves only when a score exceeds
//            it by more than 2^8 (one warp vote in the common case); probabilities go to
//            shared memory as the fp16 B operand.
//   PV       tcgen05.mma M = 128 channels of a group, N = 16 heads, K = 16 tokens, A from
//            tensor memory, accumulating O (fp32) in tensor memory; a rare rescale pass
//            multiplies O when a head's running max moves.
// Kernel B (rolaq_decode_merge): log-sum-exp merge of the per-item partials.
#pragma once
#include "common.cuh"

namespace rolaq {

constexpr int kPageTok = ROLAQ_PAGE_TOKENS;
constexpr int kPageRows = ROLAQ_PAGE_BYTES / 128;   // 144 rows of 128 B
constexpr int kTeams = 4;
constexpr int kDecodeThreads = 128 * kTeams;
constexpr int kStages = 2;                          // whole pages in flight per team
constexpr int kRing = 2;                            // TMEM A slots / P tiles per team
constexpr int kStepTok = 16;                        // tokens per step
constexpr int kRingCol = 64;                        // O: columns 0..63 (16 per group)
constexpr int kTeamCols = kRingCol + 32 * kRing;    // TMEM columns per team (ring after O)
static_assert(kTeams * kTeamCols <= 512, "tensor memory columns");
constexpr int kLutStride = 6;                       // uint2 per token row of the LUT tile
constexpr float kRescaleLog2 = 8.f;
constexpr int kMetaRow = 64;                        // page rows: codes 0..63, meta 64..79,
constexpr int kKrRow = 80;                          // RoPE keys 80..143

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
};

struct DecodeSmem {
    alignas(1024) uint8_t stage[kTeams][kStages][ROLAQ_PAGE_BYTES];
    float sT[kTeams][2][4][16][16];          // partial scores [team][buf][warp][head][token']
    alignas(128) uint8_t P[kTeams][kRing][512];   // fp16 probabilities, UMMA B layout
    alignas(16) uint2 lut[kTeams][2][kStepTok][kLutStride];   // (lo, hi) bytes of 4 x values
    float sAl[kTeams][2][16];                // rescale factor per head
    float2 team_ml[kTeams][16];
    int resc[kTeams][2];
    alignas(8) uint64_t full[kTeams][kStages];
    alignas(8) uint64_t pvbar[kTeams][kRing];
    int valid[kTeams][kStages];
    uint32_t tmem_base;
    int plan[4];
    int abort;
};
static_assert(sizeof(DecodeSmem) + 1024 <= 227 * 1024, "decode shared memory");

// ---- split plan --------------------------------------------------------------
// pages_b = ceil(L_b / 64); chunk = max(1, ceil(sum_b pages_b / target)); request b
// gets ceil(pages_b / chunk) items numbered consecutively in request order.  Executed
// by one full warp; every lane returns the same values.
struct PlanInfo { int b, first_page, n_pages, n_items, item_offset, chunk; };

__device__ __forceinline__ int plan_chunk(const int32_t* seq_lens, int batch, int target) {
    const int lane = threadIdx.x & 31;
    long long total = 0;
    for (int b = lane; b < batch; b += 32) {
        int L = max(seq_lens[b], 0);
        total += (L + kPageTok - 1) / kPageTok;
    }
    for (int o = 16; o; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    long long c = (total + target - 1) / target;
    return (int)max(1LL, c);
}

// Locate work item `item` (or request `req` when item < 0).  n_items = total item count.
__device__ PlanInfo plan_lookup(const int32_t* seq_lens, int batch, int target, int item,
                                int req) {
    const int lane = threadIdx.x & 31;
    PlanInfo pi{-1, 0, 0, 0, 0, 0};
    const int chunk = plan_chunk(seq_lens, batch, target);
    pi.chunk = chunk;
    int base = 0;
    for (int b0 = 0; b0 < batch; b0 += 32) {
        int b = b0 + lane;
        int items = 0, pages = 0;
        if (b < batch) {
            pages = (max(seq_lens[b], 0) + kPageTok - 1) / kPageTok;
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

// Instruction descriptor of the PV MMA: f16 x f16 -> f32, M = 128, N = 16.
constexpr uint32_t kPvIdesc = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
constexpr float kF16Max = 65504.f;

// Shared-memory descriptor of a K-major operand without swizzle: 8-row x 16-byte core
// matrices, K-adjacent cores 128 B apart, 8-row groups 256 B apart.
__device__ __forceinline__ uint64_t umma_desc_plain(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
           ((uint64_t)(256 >> 4) << 32) | (1ull << 46);
}
// D (tensor memory) (+)= A (tensor memory) * B (shared memory)
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d), "r"(a), "l"(bdesc), "r"(kPvIdesc), "r"(acc) : "memory");
}
// Eight fp16 pairs from one 32-bit word of codes: bytes 0-1 hold 8 codes of token A,
// bytes 2-3 8 codes of token B (code j of a byte at bits 2j).  r[k][0] = (x_A of code k
// of byte 0, x_A of code k of byte 1); r[k][1] the same for token B.  A token's lookup
// pair (lo, hi) holds the low and high bytes of its four fp16 x values, so PRMT nibbles
// c and c + 4 pick value c: the selector of a byte pair is byte * 0x11 + 0x4040 with the
// code moved to bits 0-1; __umulhi(m, 0x11 << (16 - s)) does the same for bytes 2-3
// (every multiplier fits in 32 bits).
__device__ __forceinline__ void dequant_word2(uint32_t w, uint2 la, uint2 lb, uint32_t (&r)[4][2]) {
    const uint32_t m0 = w & 0x03030303u;
    r[0][0] = prmt(la.x, la.y, m0 * 0x11u + 0x4040u);
    r[0][1] = prmt(lb.x, lb.y, __umulhi(m0, 0x11u << 16) + 0x4040u);
    const uint32_t m1 = w & 0x0C0C0C0Cu;
    r[1][0] = prmt(la.x, la.y, (m1 >> 2) * 0x11u + 0x4040u);
    r[1][1] = prmt(lb.x, lb.y, __umulhi(m1, 0x11u << 14) + 0x4040u);
    const uint32_t m2 = w & 0x30303030u;
    r[2][0] = prmt(la.x, la.y, (m2 >> 4) * 0x11u + 0x4040u);
    r[2][1] = prmt(lb.x, lb.y, __umulhi(m2, 0x11u << 12) + 0x4040u);
    const uint32_t m3 = w & 0xC0C0C0C0u;
    r[3][0] = prmt(la.x, la.y, __umulhi(m3, 0x11u << 26) + 0x4040u);
    r[3][1] = prmt(lb.x, lb.y, __umulhi(m3, 0x11u << 10) + 0x4040u);
}

// Issue the bulk copy of one page (all 144 rows) into stage k % kStages, or mark the
// stage invalid when the page-table entry is outside the pool.
__device__ __forceinline__ void load_page(DecodeSmem& sm, const CUtensorMap* map, const DecodeArgs& args,
                                          int team, int b, int page_idx, int k) {
    const int st = k % kStages;
    long long pid = -1;
    if (page_idx < args.max_pages) pid = args.page_table[(long long)b * args.max_pages + page_idx];
    const uint32_t bar = smem_u32(&sm.full[team][st]);
    if (pid >= 0 && pid < args.num_pages) {
        sm.valid[team][st] = 1;
        mbar_arrive_expect_tx(bar, ROLAQ_PAGE_BYTES);
        tma_load_2d(smem_u32(sm.stage[team][st]), map, 0, (int)(pid * kPageRows), bar);
    } else {
        sm.valid[team][st] = 0;
        raise_status(ROLAQ_STATUS_BAD_PAGE);
        mbar_arrive(bar);
    }
}

// Lookup pair of token tt (0..15 of step `sub` of a staged page), group gg: fp16 of
// mean + scale * (-b, -a, a, b), split into low bytes and high bytes.  Tokens past the
// sequence end or on an invalid page get zeros, so their x is 0 (their scores are masked).
// Values beyond the fp16 range raise ROLAQ_STATUS_RANGE.
__device__ __forceinline__ void lut_prep(const uint8_t* pg, bool vpage, int sub, int tt, int gg, int pos,
                                         int L, float la, float lb, uint2* lut) {
    uint2 v = make_uint2(0u, 0u);
    if (vpage && pos < L) {
        const int pt = kStepTok * sub + tt;
        const float2 ms = *reinterpret_cast<const float2*>(
            pg + swz128(kMetaRow + (pt >> 2), (pt & 3) * 32 + 8 * gg));
        if (!(fabsf(ms.x) + fabsf(ms.y) * lb < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
        const uint32_t w01 = pack_f16(fmaf(ms.y, -lb, ms.x), fmaf(ms.y, -la, ms.x));
        const uint32_t w23 = pack_f16(fmaf(ms.y, la, ms.x), fmaf(ms.y, lb, ms.x));
        v.x = prmt(w01, w23, 0x6420u);
        v.y = prmt(w01, w23, 0x7531u);
    }
    lut[tt * kLutStride + gg] = v;
}

// Per-thread byte offsets inside a staged page, fixed for the whole kernel: every step's
// code and RoPE rows start at a multiple of 8, so the 128-byte swizzle of a thread's
// position does not depend on the step (step sub adds 2048, the second n-tile 1024).
struct StageOffsets {
    uint32_t code[4];      // codes of token r, channels 32q + 8i.. of group g
    uint32_t kr0, kr1;     // RoPE channels 16q + 2i.. and 16q + 8 + 2i.. of token r
};
__device__ __forceinline__ StageOffsets stage_offsets(int q, int r, int i) {
    StageOffsets o;
#pragma unroll
    for (int g = 0; g < 4; ++g)
        o.code[g] = r * 128 + (((2 * g + (q >> 1)) ^ r) << 4) + ((8 * q + 2 * i) & 15);
    o.kr0 = (kKrRow + r) * 128 + (((2 * q) ^ r) << 4) + 4 * i;
    o.kr1 = (kKrRow + r) * 128 + (((2 * q + 1) ^ r) << 4) + 4 * i;
    return o;
}

// QK of one 16-token step for warp q, one channel group at a time.  Thread (r, i) builds
// the x fragments of tokens r and r + 8 for channels 32q + 8i .. 32q + 8i + 7 of group g:
// x[ks][nt][h] holds B-fragment k indices 2i + 8h + {0,1} of k-slice ks, which are
// channels 32q + 8i + 2ks + h + {0, 4} (the query fragments use the same order).  Right
// after its MMAs each group's fragments are transposed and stored as the PV A operand
// (lanes 32q + 16ks + y for B-fragment k index y; ring columns 8g + c, where column 2i
// holds tokens (2i, 2i+1) and column 2i + 1 tokens (8 + 2i, 9 + 2i)); the ring slot is
// waited for before the first store.  Scores of the 16 heads x 16 tokens over this warp's
// channels (plus its RoPE channels) go to sT with the token index XOR 8 * ((head >> 1) & 1)
// (conflict-free stores and loads).  `pg` points at the step's first row.  PROT: some
// token of the step is protected and takes its x from the bf16 side store (as fp16).
template <bool PROT>
__device__ __forceinline__ void qk_step(const uint8_t* pg, const StageOffsets& so, const uint2* lut,
                                        float (*sT)[16], int q, int r, int i, const uint32_t (&qa)[4][2][4],
                                        const uint32_t (&qra)[4], uint32_t a_taddr, uint32_t slot_bar,
                                        unsigned slot_parity, bool slot_wait, volatile int* abort, int pos0,
                                        int L, int recent_start, const DecodeArgs& args, int b) {
    bool pa = false, pb = false;
    const uint4* srca = nullptr;
    const uint4* srcb = nullptr;
    if (PROT) {
        const int nslot = args.n_sink + args.n_recent;
        const int p0 = pos0 + r, p1 = pos0 + 8 + r;
        pa = p0 < L && (p0 < args.n_sink || p0 >= recent_start);
        pb = p1 < L && (p1 < args.n_sink || p1 >= recent_start);
        const int s0 = p0 < args.n_sink ? p0 : args.n_sink + p0 % max(args.n_recent, 1);
        const int s1 = p1 < args.n_sink ? p1 : args.n_sink + p1 % max(args.n_recent, 1);
        srca = reinterpret_cast<const uint4*>(args.prot + ((size_t)b * nslot + s0) * ROLAQ_D_C + 32 * q + 8 * i);
        srcb = reinterpret_cast<const uint4*>(args.prot + ((size_t)b * nslot + s1) * ROLAQ_D_C + 32 * q + 8 * i);
    }
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t c0 = *reinterpret_cast<const uint16_t*>(pg + so.code[g]);
        const uint32_t c1 = *reinterpret_cast<const uint16_t*>(pg + so.code[g] + 1024);
        uint32_t t[4][2];
        dequant_word2(c0 | (c1 << 16), lut[r * kLutStride + g], lut[(r + 8) * kLutStride + g], t);
        uint32_t x[2][2][2];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) x[ks][nt][h] = t[2 * ks + h][nt];
        if (PROT) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (nt == 0 ? pa : pb) {
                    const uint4 u = (nt == 0 ? srca : srcb)[16 * g];
                    x[0][nt][0] = pack_f16(bf16_lo(u.x), bf16_lo(u.z));
                    x[0][nt][1] = pack_f16(bf16_hi(u.x), bf16_hi(u.z));
                    x[1][nt][0] = pack_f16(bf16_lo(u.y), bf16_lo(u.w));
                    x[1][nt][1] = pack_f16(bf16_hi(u.y), bf16_hi(u.w));
                }
            }
        }
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma_f16_16816(acc[nt], qa[g][ks], x[ks][nt][0], x[ks][nt][1]);
        if (g == 0) {
            if (slot_wait) mbar_wait(slot_bar, slot_parity, abort);
            tc_fence_after();
        }
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const uint32_t v0 = movmatrix_trans(x[ks][0][0]);
            const uint32_t v1 = movmatrix_trans(x[ks][1][0]);
            const uint32_t v2 = movmatrix_trans(x[ks][0][1]);
            const uint32_t v3 = movmatrix_trans(x[ks][1][1]);
            asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1, %2, %3, %4};"
                         :: "r"(a_taddr + ((uint32_t)(16 * ks) << 16) + 8 * g), "r"(v0), "r"(v1), "r"(v2),
                            "r"(v3)
                         : "memory");
        }
    }
    const int sw = 8 * ((r >> 1) & 1);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        // RoPE part of the score for channels 16q..16q+15
        const uint32_t kb0 = *reinterpret_cast<const uint32_t*>(pg + so.kr0 + 1024 * nt);
        const uint32_t kb1 = *reinterpret_cast<const uint32_t*>(pg + so.kr1 + 1024 * nt);
        mma_bf16_16816(acc[nt], qra, kb0, kb1);
        const int t = (8 * nt + 2 * i) ^ sw;
        *reinterpret_cast<float2*>(&sT[r][t]) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(&sT[r + 8][t]) = make_float2(acc[nt][2], acc[nt][3]);
    }
}

// Softmax of one step for head hh (of the 16-head chunk), tokens 2jj, 2jj+1.  The
// reference max m_ref moves only when a score exceeds it by more than kRescaleLog2
// (one warp vote in the common case), so probabilities relative to m_ref stay below
// 2^kRescaleLog2.  The fp16 probabilities go to the B tile at K positions
// 4jj, 4jj+1 (jj < 4) or 4(jj-4)+2, +3, matching the A tile's column order.
__device__ __forceinline__ void softmax_step(const float (*sT)[16][16], uint8_t* Pt, float* sAl, int* resc,
                                             int hh, int jj, int nvalid, float scale_log2, bool first,
                                             float& m_ref, float& l_part) {
    const int t = (2 * jj) ^ (8 * ((hh >> 1) & 1));
    const float2 v0 = *reinterpret_cast<const float2*>(&sT[0][hh][t]);
    const float2 v1 = *reinterpret_cast<const float2*>(&sT[1][hh][t]);
    const float2 v2 = *reinterpret_cast<const float2*>(&sT[2][hh][t]);
    const float2 v3 = *reinterpret_cast<const float2*>(&sT[3][hh][t]);
    float s0 = ((v0.x + v1.x) + (v2.x + v3.x)) * scale_log2;
    float s1 = ((v0.y + v1.y) + (v2.y + v3.y)) * scale_log2;
    if (2 * jj >= nvalid) s0 = -INFINITY;
    if (2 * jj + 1 >= nvalid) s1 = -INFINITY;
    float alpha = 1.f;
    const bool up = fmaxf(s0, s1) > m_ref + kRescaleLog2 || (m_ref == -INFINITY && fmaxf(s0, s1) > -INFINITY);
    if (__any_sync(0xffffffffu, up)) {
        float pm = fmaxf(s0, s1);
        pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 1));
        pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 2));
        pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 4));
        if (pm > m_ref + kRescaleLog2 || (m_ref == -INFINITY && pm > -INFINITY)) {
            alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - pm);
            m_ref = pm;
            l_part *= alpha;
        }
    }
    const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
    const float p0 = ex2(s0 - mu), p1 = ex2(s1 - mu);
    l_part += p0 + p1;
    const int kp = jj < 4 ? 4 * jj : 4 * (jj - 4) + 2;
    const int off = (hh >> 3) * 256 + (kp >> 3) * 128 + (hh & 7) * 16 + (kp & 7) * 2;
    *reinterpret_cast<uint32_t*>(Pt + off) = pack_f16(p0, p1);
    if (jj == 0) sAl[hh] = alpha;
    if (alpha != 1.f && !first) *resc = 1;
}

// PV of team step jp, called by all 128 threads of the team after the step barrier that
// follows softmax(jp).  When some head's running max moved at jp, every warp first scales
// its lanes of O (the PV of step jp-1 has completed: its ring slot was waited for), then
// lane 0 of the team's first warp issues the four group MMAs and commits them to the
// slot's barrier.
__device__ __forceinline__ void pv_issue(DecodeSmem& sm, int team, int q, int lane, int jp, uint32_t tmem,
                                         int bar_id) {
    const int buf = jp & 1;
    if (sm.resc[team][buf]) {
        tc_fence_after();
        const uint32_t ocol = tmem + ((uint32_t)(32 * q) << 16) + team * kTeamCols;
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
            uint32_t u[16];
            tmem_ld16(ocol + 16 * g, u);
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < 16; ++h) u[h] = __float_as_uint(__uint_as_float(u[h]) * sm.sAl[team][buf][h]);
            tmem_st16(ocol + 16 * g, u);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar_sync(bar_id, 128);
        if (q == 0 && lane == 0) sm.resc[team][buf] = 0;
    }
    if (q == 0 && lane == 0) {
        tc_fence_after();
        const int slot = jp % kRing;
        const uint32_t obase = tmem + team * kTeamCols;
        const uint32_t abase = obase + kRingCol + 32 * slot;
        const uint64_t bd = umma_desc_plain(smem_u32(sm.P[team][slot]));
#pragma unroll
        for (int g = 0; g < 4; ++g) umma_ts(obase + 16 * g, abase + 8 * g, bd, jp > 0 ? 1u : 0u);
        umma_commit(smem_u32(&sm.pvbar[team][slot]));
    }
}

__global__ void __launch_bounds__(kDecodeThreads, 1)
rolaq_decode_split(const __grid_constant__ CUtensorMap map_page, const DecodeArgs args) {
    extern __shared__ uint8_t smem_raw[];
    // offset the __shared__ array itself (not an integer address) so that every access
    // stays a shared-memory access
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
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
        for (int t = 0; t < kTeams; ++t) {
            for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&sm.full[t][s]), 1);
            for (int s = 0; s < kRing; ++s) mbar_init(smem_u32(&sm.pvbar[t][s]), 1);
            sm.resc[t][0] = sm.resc[t][1] = 0;
        }
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_page);
    }
    __syncthreads();
    const int b = sm.plan[0];
    if (b < 0) return;                         // item past the end of the plan
    const int first_page = sm.plan[1], n_pages = sm.plan[2];
    const int L = args.seq_lens[b];
    const int team = warp >> 2, q = warp & 3;
    const int tid = threadIdx.x & 127;
    const bool leader = (q == 0) && (lane == 0);
    const int n_team = n_pages > team ? (n_pages - team + kTeams - 1) / kTeams : 0;
    const int J = n_team * (kPageTok / kStepTok);
    auto page_of = [&](int k) { return first_page + team + kTeams * k; };
    if (leader)
        for (int k = 0; k < n_team && k < kStages; ++k) load_page(sm, &map_page, args, team, b, page_of(k), k);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                     :: "r"(smem_u32(&sm.tmem_base)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }

    const int r = lane >> 2, i = lane & 3;     // mma fragment row group / thread in group
    const int h0 = hc * 16;
    // Query fragments (fp16) in the channel order of qk_step.
    uint32_t qa[4][2][4];
    {
        const uint16_t* u0 = reinterpret_cast<const uint16_t*>(args.q + ((size_t)b * args.heads + h0 + r) * ROLAQ_D_C);
        const uint16_t* u1 = u0 + 8 * ROLAQ_D_C;
        float qmax = 0.f;
        auto f = [&](const uint16_t* u, int c) {
            const float v = __uint_as_float((uint32_t)u[c] << 16);
            qmax = fmaxf(qmax, fabsf(v));
            return v;
        };
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int c = 128 * g + 32 * q + 8 * i + 2 * ks;
                qa[g][ks][0] = pack_f16(f(u0, c), f(u0, c + 4));
                qa[g][ks][1] = pack_f16(f(u1, c), f(u1, c + 4));
                qa[g][ks][2] = pack_f16(f(u0, c + 1), f(u0, c + 5));
                qa[g][ks][3] = pack_f16(f(u1, c + 1), f(u1, c + 5));
            }
        if (!(qmax < kF16Max)) raise_status(ROLAQ_STATUS_RANGE);
    }
    uint32_t qra[4];
    {
        const uint32_t* r0 = reinterpret_cast<const uint32_t*>(
            args.qr + ((size_t)b * args.heads + h0 + r) * ROLAQ_D_R + 16 * q);
        const uint32_t* r1 = r0 + 8 * ROLAQ_D_R / 2;
        qra[0] = r0[i];
        qra[1] = r1[i];
        qra[2] = r0[4 + i];
        qra[3] = r1[4 + i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int hh = 4 * q + (lane >> 3), jj = lane & 7;   // softmax: head, token pair
    const int bar_id = 1 + team;
    const bool protect = args.n_sink > 0 || args.n_recent > 0;
    const int recent_start = L - args.n_recent;
    const float lva = args.level_a, lvb = args.level_b;
    const uint32_t a_lane = tmem + ((uint32_t)(32 * q) << 16) + team * kTeamCols + kRingCol;
    const StageOffsets so = stage_offsets(q, r, i);
    float m_ref = -INFINITY, l_part = 0.f;

    if (J > 0 && tid < 64) {
        mbar_wait(smem_u32(&sm.full[team][0]), 0, &sm.abort);
        lut_prep(sm.stage[team][0], sm.valid[team][0] != 0, 0, tid >> 2, tid & 3,
                 page_of(0) * kPageTok + (tid >> 2), L, lva, lvb, &sm.lut[team][0][0][0]);
    }
    named_bar_sync(bar_id, 128);

    for (int j = 0; j < J; ++j) {
        const int k = j >> 2, sub = j & 3, st = k % kStages;
        if (sub == 0) mbar_wait(smem_u32(&sm.full[team][st]), (k / kStages) & 1, &sm.abort);
        const uint8_t* pg = sm.stage[team][st];
        const int pos0 = page_of(k) * kPageTok + kStepTok * sub;
        const int nvalid = sm.valid[team][st] ? min(max(L - pos0, 0), kStepTok) : 0;
        const bool prot = protect && (pos0 < args.n_sink || pos0 + kStepTok > recent_start);
        const int slot = j % kRing;
        const uint32_t slot_bar = smem_u32(&sm.pvbar[team][slot]);
        const unsigned slot_par = (unsigned)(((j - kRing) / kRing) & 1);
        const uint8_t* pgs = pg + sub * (kStepTok * 128);
        // QK of step j; its A tile goes to ring slot j % kRing once PV(j - kRing) has read it
        if (prot)
            qk_step<true>(pgs, so, &sm.lut[team][j & 1][0][0], sm.sT[team][j & 1][q], q, r, i, qa, qra,
                          a_lane + 32 * slot, slot_bar, slot_par, j >= kRing, &sm.abort, pos0, L, recent_start,
                          args, b);
        else
            qk_step<false>(pgs, so, &sm.lut[team][j & 1][0][0], sm.sT[team][j & 1][q], q, r, i, qa, qra,
                           a_lane + 32 * slot, slot_bar, slot_par, j >= kRing, &sm.abort, pos0, L, recent_start,
                           args, b);
        tmem_st_wait();
        tc_fence_before();
        // lookup pairs of step j + 1
        if (j + 1 < J && tid < 64) {
            const int jn = j + 1, kn = jn >> 2, subn = jn & 3, stn = kn % kStages;
            if (subn == 0) mbar_wait(smem_u32(&sm.full[team][stn]), (kn / kStages) & 1, &sm.abort);
            lut_prep(sm.stage[team][stn], sm.valid[team][stn] != 0, subn, tid >> 2, tid & 3,
                     page_of(kn) * kPageTok + kStepTok * subn + (tid >> 2), L, lva, lvb,
                     &sm.lut[team][jn & 1][0][0]);
        }
        named_bar_sync(bar_id, 128);
        // page k is fully read after its last step: refill its stage
        if (leader && sub == 3 && k + kStages < n_team)
            load_page(sm, &map_page, args, team, b, page_of(k + kStages), k + kStages);
        if (j >= 1) pv_issue(sm, team, q, lane, j - 1, tmem, bar_id);
        softmax_step(sm.sT[team][j & 1], sm.P[team][slot], sm.sAl[team][j & 1], &sm.resc[team][j & 1], hh, jj,
                     nvalid, args.scale_log2, j == 0, m_ref, l_part);
        fence_proxy_async_smem();
    }
    if (J > 0) {
        if (J >= kRing) mbar_wait(smem_u32(&sm.pvbar[team][J % kRing]), ((J - kRing) / kRing) & 1, &sm.abort);
        named_bar_sync(bar_id, 128);
        pv_issue(sm, team, q, lane, J - 1, tmem, bar_id);
        mbar_wait(smem_u32(&sm.pvbar[team][(J - 1) % kRing]), ((J - 1) / kRing) & 1, &sm.abort);
        tc_fence_after();
    }
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 4);
    if (jj == 0) sm.team_ml[team][hh] = make_float2(m_ref, l_part);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- merge the teams: warp q of team t writes channel groups t, t + kTeams, ... ----
    {
        float Mx[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            float m = sm.team_ml[0][h].x;
#pragma unroll
            for (int t = 1; t < kTeams; ++t) m = fmaxf(m, sm.team_ml[t][h].x);
            Mx[h] = m;
        }
        const int ks = lane >> 4, y = lane & 15;
        const int chq = 32 * q + 8 * ((y & 7) >> 1) + 4 * (y & 1) + 2 * ks + (y >> 3);
#pragma unroll 1
        for (int g = team; g < 4; g += kTeams) {
            float acc[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) acc[h] = 0.f;
#pragma unroll 1
            for (int t = 0; t < kTeams; ++t) {
                float w[16];
                bool any = false;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const float m = sm.team_ml[t][h].x;
                    w[h] = (m == -INFINITY) ? 0.f : ex2(m - Mx[h]);
                    any |= w[h] != 0.f;
                }
                if (any) {                           // the same for every lane of the warp
                    uint32_t u[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + t * kTeamCols + 16 * g, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 16; ++h)
                        if (w[h] != 0.f) acc[h] = fmaf(w[h], __uint_as_float(u[h]), acc[h]);
                }
            }
            float* dst = args.ws_o + ((size_t)blockIdx.x * args.heads + h0) * ROLAQ_D_C + 128 * g + chq;
#pragma unroll
            for (int h = 0; h < 16; ++h) dst[(size_t)h * ROLAQ_D_C] = acc[h];
        }
        if (team == 0 && q == 0 && lane < 16) {
            float m = sm.team_ml[0][lane].x;
            for (int t = 1; t < kTeams; ++t) m = fmaxf(m, sm.team_ml[t][lane].x);
            float l = 0.f;
            for (int t = 0; t < kTeams; ++t) {
                const float2 ml = sm.team_ml[t][lane];
                if (ml.x != -INFINITY) l += ex2(ml.x - m) * ml.y;
            }
            args.ws_ml[(size_t)blockIdx.x * args.heads + h0 + lane] = make_float2(m, l);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" :: "r"(tmem) : "memory");
    }
}

// ---- merge --------------------------------------------------------------------
// grid (batch, heads), 512 threads: out[b,h,:] = sum_i w_i o_i / sum_i w_i l_i with
// w_i = 2^(m_i - max m); lse = (max m + log2(sum w l)) * ln 2.  Warp w takes partials
// w, w + 16, ...; lane l owns channels 4l + 128j (j = 0..3), so every thread keeps many
// independent loads in flight; the 16 warp sums are added through shared memory.
constexpr int kMergeThreads = 512;

__global__ void __launch_bounds__(kMergeThreads)
rolaq_decode_merge(const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
                   const int32_t* seq_lens, int batch, int heads, int target,
                   float* __restrict__ out, float* __restrict__ lse) {
    __shared__ int s_plan[2];
    __shared__ float s_red[kMergeThreads / 32];
    __shared__ float s_M, s_den;
    __shared__ __align__(16) float s_acc[kMergeThreads / 32][ROLAQ_D_C];
    const int b = blockIdx.x, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kWarps = kMergeThreads / 32;
    if (warp == 0) {
        PlanInfo pi = plan_lookup(seq_lens, batch, target, -1, b);
        if (lane == 0) { s_plan[0] = pi.item_offset; s_plan[1] = pi.n_items; }
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
        float m = -INFINITY;
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
    if (threadIdx.x == 0) {
        float dsum = 0.f;
        for (int w = 0; w < kWarps; ++w) dsum += s_red[w];
        s_den = dsum;
    }
    __syncthreads();
    den = s_den;
    const int c = threadIdx.x;               // one output channel per thread
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += s_acc[w][c];
    out[((size_t)b * heads + h) * ROLAQ_D_C + c] = den > 0.f ? v / den : 0.f;
    if (lse && threadIdx.x == 0)
        lse[(size_t)b * heads + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace rolaq
