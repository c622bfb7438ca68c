// Absorbed-MLA decode attention over the packed 2-bit cache ("RoLaQ", §2.1, §3.3):
// scores (q_c_rot . x + q_R . k_R) * sm_scale with x = mean + scale * level(code),
// softmax over the request's tokens, 512-d latent readout in the rotated basis.
//
// Kernel A (rolaq_decode_split): one CTA per (work item, 16-head chunk).  A work item is a
// run of whole pages of one request (split-K over the sequence).  8 warps in two teams of
// four.  Team t owns tokens 32t..32t+31 of every page: lane 0 of its warp 0 issues the
// bulk tensor copies of that half page (codes, metadata, RoPE rows; 128-byte swizzle)
// into the team's ring of shared-memory stages, and the team keeps its own online-softmax
// state.  Inside a team, warp g owns content-channel group g (128 channels) and RoPE
// channels 16g..16g+15.
//
// A team walks its tokens in steps of 16 as a software pipeline with one team barrier per
// step: QK(j+1) | barrier | softmax(j+1) and PV(j).
//   QK    mma.sync m16n8k16 (heads = M) on bf16 level fragments built in registers from
//         the codes (PRMT lookup); the group metadata is folded outside the MMA
//         (q.x = mean * sum(q_g) + scale * (q_g . level)); partial scores per group go to
//         shared memory.
//   softmax  warp g sums the four partials for heads 4g..4g+3; the running max moves only
//         when a score exceeds it by more than 2^8 (checked with one warp vote), so the
//         common step has no shuffles; row sums stay per lane until the end.
//   PV    the same level fragments transposed in registers (movmatrix), the scale folded
//         into P, the mean term kept as a per-head rank-1 accumulator.
// Kernel B (rolaq_decode_merge): log-sum-exp merge of the per-(item, team) partials.
#pragma once
#include "common.cuh"

namespace rolaq {

constexpr int kPageTok = ROLAQ_PAGE_TOKENS;
constexpr int kPageRows = ROLAQ_PAGE_BYTES / 128;   // 144 rows of 128 B
constexpr int kNStage = 8;                          // half-page stages per team
constexpr int kStepTok = 16;                        // tokens per pipeline step
constexpr int kSStride = 24;                        // floats per head row of sT / sP
constexpr int kDecodeThreads = 256;
constexpr float kRescaleLog2 = 8.f;
// A team stages its half of a page: 32 code rows, 8 metadata rows, 32 RoPE rows.
constexpr int kHalfBytes = 9216;
constexpr int kHalfMetaOff = 4096;                  // smem row 32
constexpr int kHalfKrOff = 5120;                    // smem row 40

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
    uint32_t lut_lo, lut_hi;     // low / high bytes of the four bf16 levels / kappa
    float kappa;                 // level = kappa * bf16 level
    int target_items;
    float* ws_o;                 // [items][2][heads][512]
    float2* ws_ml;               // [items][2][heads]  (reference max (log2 units), sum)
};

struct DecodeSmem {
    alignas(1024) uint8_t stage[2][kNStage][kHalfBytes];
    float sT[2][2][4][16][kSStride];     // [team][buffer][group][head][token]
    float sP[2][2][16][kSStride];        // [team][buffer][head][token]
    float sAl[2][2][16];                 // [team][buffer][head] rescale factor
    alignas(8) uint64_t full[2][kNStage];
    int valid[2][kNStage];
    int plan[4];
    int abort;
};

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

// Channel (within a 128-channel group) that QK k-slice s, MMA k index kk maps to.
// Thread i = lane % 4 loads code bytes 8i..8i+7 of the group; its fragment values are
// channels 32i + 16*(s/4) + 8*(kk/8) + 4*(kk%2) + s%4 (any channel order works for a
// dot product as long as the query fragments follow it).
__device__ __forceinline__ int qk_channel(int s, int kk) {
    return 32 * ((kk & 7) >> 1) + 16 * (s >> 2) + 8 * (kk >> 3) + 4 * (kk & 1) + (s & 3);
}

// Four bf16 level pairs from one 32-bit word of codes (16 codes, 2 bit each).
// Output r[k][0] = (level(code k), level(code 4+k)), r[k][1] = (code 8+k, code 12+k).
// Selector byte for code c is c | (c + 4) << 4: PRMT takes the low level byte from
// lut_lo[c] and the high byte from lut_hi[c].  (m >> 2k) * 0x11 spreads the code in each
// byte to both nibbles; __umulhi(m, 0x11 << (16 - 2k)) does the same and moves bytes 2..3
// down to 0..1 (every multiplier must fit in 32 bits).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t lo, uint32_t hi,
                                             uint32_t (&r)[4][2]) {
    uint32_t m0 = w & 0x03030303u;
    r[0][0] = prmt(lo, hi, m0 * 0x11u + 0x40404040u);
    r[0][1] = prmt(lo, hi, __umulhi(m0, 0x11u << 16) + 0x4040u);
    uint32_t m1 = w & 0x0C0C0C0Cu;
    r[1][0] = prmt(lo, hi, (m1 >> 2) * 0x11u + 0x40404040u);
    r[1][1] = prmt(lo, hi, __umulhi(m1, 0x11u << 14) + 0x4040u);
    uint32_t m2 = w & 0x30303030u;
    r[2][0] = prmt(lo, hi, (m2 >> 4) * 0x11u + 0x40404040u);
    r[2][1] = prmt(lo, hi, __umulhi(m2, 0x11u << 12) + 0x4040u);
    uint32_t m3 = w & 0xC0C0C0C0u;
    r[3][0] = prmt(lo, hi, __umulhi(m3, 0x11u << 26) + 0x40404040u);
    r[3][1] = prmt(lo, hi, __umulhi(m3, 0x11u << 10) + 0x4040u);
}

// Issue the three copies of one team's half of page `page_idx` into stage k % kNStage
// (or mark it invalid when the page-table entry is outside the pool).
__device__ __forceinline__ void load_half_page(DecodeSmem& sm, const CUtensorMap* map32,
                                               const CUtensorMap* map8, const DecodeArgs& args,
                                               int team, int b, int page_idx, int k) {
    const int st = k % kNStage;
    long long pid = -1;
    if (page_idx < args.max_pages) pid = args.page_table[(long long)b * args.max_pages + page_idx];
    const uint32_t bar = smem_u32(&sm.full[team][st]);
    if (pid >= 0 && pid < args.num_pages) {
        sm.valid[team][st] = 1;
        const int row0 = (int)(pid * kPageRows);
        const uint32_t dst = smem_u32(sm.stage[team][st]);
        mbar_arrive_expect_tx(bar, kHalfBytes);
        tma_load_2d(dst, map32, 0, row0 + 32 * team, bar);
        tma_load_2d(dst + kHalfMetaOff, map8, 0, row0 + 64 + 8 * team, bar);
        tma_load_2d(dst + kHalfKrOff, map32, 0, row0 + 80 + 32 * team, bar);
    } else {
        sm.valid[team][st] = 0;
        raise_status(ROLAQ_STATUS_BAD_PAGE);
        mbar_arrive(bar);
    }
}

// Per-warp state of a team's pipeline.
struct StepRegs {
    uint32_t bq[2][8][2];    // level fragments of the step's two n-tiles (8 tokens each)
    float mu[2][2], sc[2][2];  // mean and kappa*scale of the fragment-column tokens
};

// QK for one 16-token step (rows 16*sub.. of the staged half page) and this warp's group:
// dequantise, MMA, fold the metadata, add the RoPE part, store the partial scores.
// FULL: all 16 tokens are in the sequence and none is protected.
template <bool FULL>
__device__ __forceinline__ void qk_step(const uint8_t* pg, int sub, float (*sT)[kSStride], int r, int i,
                                        int g, uint32_t lut_lo, uint32_t lut_hi, float kappa,
                                        const uint32_t (&qa)[8][4], const uint32_t (&qra)[4],
                                        float qs0, float qs1, int nvalid, int pos0, int L,
                                        int recent_start, const DecodeArgs& args, int b, StepRegs& s) {
    const int row0 = 16 * sub;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const uint2 w = *reinterpret_cast<const uint2*>(pg + swz128(row0 + 8 * nt + r, 32 * g + 8 * i));
        uint32_t t[4][2];
        dequant_word(w.x, lut_lo, lut_hi, t);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) { s.bq[nt][kk][0] = t[kk][0]; s.bq[nt][kk][1] = t[kk][1]; }
        dequant_word(w.y, lut_lo, lut_hi, t);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) { s.bq[nt][4 + kk][0] = t[kk][0]; s.bq[nt][4 + kk][1] = t[kk][1]; }
    }
    if (!FULL) {
        // Protected tokens read their bf16 rotated content instead of the codes.
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int pos = pos0 + 8 * nt + r;
            if (pos < L && (pos < args.n_sink || pos >= recent_start)) {
                const int slot = pos < args.n_sink ? pos : args.n_sink + pos % args.n_recent;
                const uint4* src = reinterpret_cast<const uint4*>(
                    args.prot + ((size_t)b * (args.n_sink + args.n_recent) + slot) * ROLAQ_D_C + 128 * g + 32 * i);
                uint32_t wv[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 v = src[q4];
                    wv[4 * q4 + 0] = v.x; wv[4 * q4 + 1] = v.y; wv[4 * q4 + 2] = v.z; wv[4 * q4 + 3] = v.w;
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int base = 16 * (ks >> 2), kk = ks & 3;
                    const uint32_t sel = (kk & 1) ? 0x7632u : 0x5410u;
                    s.bq[nt][ks][0] = prmt(wv[(base + kk) >> 1], wv[(base + 4 + kk) >> 1], sel);
                    s.bq[nt][ks][1] = prmt(wv[(base + 8 + kk) >> 1], wv[(base + 12 + kk) >> 1], sel);
                }
            }
        }
    }
    // metadata of the two tokens in each n-tile's column pair: mean, scale (kappa folded in)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = row0 + 8 * nt + 2 * i + e;        // token row in the half page
            const float2 ms = *reinterpret_cast<const float2*>(pg + swz128(32 + (t >> 2), (t & 3) * 32 + 8 * g));
            if (FULL) {
                s.mu[nt][e] = ms.x;
                s.sc[nt][e] = ms.y * kappa;
            } else {
                const int tl = 8 * nt + 2 * i + e;
                const int pos = pos0 + tl;
                const bool valid = tl < nvalid;
                const bool prot = pos < args.n_sink || pos >= recent_start;
                s.mu[nt][e] = (valid && !prot) ? ms.x : 0.f;
                s.sc[nt][e] = valid ? (prot ? 1.f : ms.y * kappa) : 0.f;
            }
        }
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_bf16_16816(acc[nt], qa[ks], s.bq[nt][ks][0], s.bq[nt][ks][1]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        // fold the group metadata: q.x = mean * sum(q_g) + scale * (q_g . level)
        acc[nt][0] = fmaf(s.sc[nt][0], acc[nt][0], s.mu[nt][0] * qs0);
        acc[nt][1] = fmaf(s.sc[nt][1], acc[nt][1], s.mu[nt][1] * qs0);
        acc[nt][2] = fmaf(s.sc[nt][0], acc[nt][2], s.mu[nt][0] * qs1);
        acc[nt][3] = fmaf(s.sc[nt][1], acc[nt][3], s.mu[nt][1] * qs1);
        // RoPE part of the score for channels 16g..16g+15
        const int row = 40 + row0 + 8 * nt + r;
        const uint32_t kb0 = *reinterpret_cast<const uint32_t*>(pg + swz128(row, 32 * g + 4 * i));
        const uint32_t kb1 = *reinterpret_cast<const uint32_t*>(pg + swz128(row, 32 * g + 16 + 4 * i));
        mma_bf16_16816(acc[nt], qra, kb0, kb1);
        const int tl = 8 * nt + 2 * i;
        if (!FULL) {
            if (tl >= nvalid) { acc[nt][0] = -INFINITY; acc[nt][2] = -INFINITY; }
            if (tl + 1 >= nvalid) { acc[nt][1] = -INFINITY; acc[nt][3] = -INFINITY; }
        }
        *reinterpret_cast<float2*>(&sT[r][tl]) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(&sT[r + 8][tl]) = make_float2(acc[nt][2], acc[nt][3]);
    }
}

// Softmax for heads 4g..4g+3 over one step's 16 tokens: lane (head hh, token pair jj).
// The reference max m_ref moves only when a score exceeds it by more than kRescaleLog2
// (one warp vote in the common case; shuffles only when some head moves), so the
// probabilities relative to m_ref stay below 2^kRescaleLog2.  l_part is this lane's share
// of the row sum, reduced over the 8 lanes of the head at the end.
__device__ __forceinline__ void softmax_step(float (*sT)[16][kSStride], float (*sP)[kSStride], float* sAl,
                                             int hh, int jj, float scale_log2, float& m_ref, float& l_part) {
    float2 v0 = *reinterpret_cast<const float2*>(&sT[0][hh][2 * jj]);
    float2 v1 = *reinterpret_cast<const float2*>(&sT[1][hh][2 * jj]);
    float2 v2 = *reinterpret_cast<const float2*>(&sT[2][hh][2 * jj]);
    float2 v3 = *reinterpret_cast<const float2*>(&sT[3][hh][2 * jj]);
    const float s0 = ((v0.x + v1.x) + (v2.x + v3.x)) * scale_log2;
    const float s1 = ((v0.y + v1.y) + (v2.y + v3.y)) * scale_log2;
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
    *reinterpret_cast<float2*>(&sP[hh][2 * jj]) = make_float2(p0, p1);
    if (jj == 0) sAl[hh] = alpha;
}

// PV inputs of one step (probabilities of the fragment rows/columns, rescale factors),
// read before the softmax of the next step writes its own buffers.
struct PvIn {
    float2 p00, p10, p02, p12;
    float al0, al1;
};
__device__ __forceinline__ PvIn pv_load(const float (*__restrict__ sP)[kSStride], const float* __restrict__ sAl,
                                        int r, int i) {
    PvIn v;
    const int tl = 2 * i;
    v.p00 = *reinterpret_cast<const float2*>(&sP[r][tl]);
    v.p10 = *reinterpret_cast<const float2*>(&sP[r + 8][tl]);
    v.p02 = *reinterpret_cast<const float2*>(&sP[r][tl + 8]);
    v.p12 = *reinterpret_cast<const float2*>(&sP[r + 8][tl + 8]);
    v.al0 = sAl[r];
    v.al1 = sAl[r + 8];
    return v;
}

// PV for one step: O_g[h, ch] += sum_t p * scale_t * level + (sum_t p * mean_t).
__device__ __forceinline__ void pv_step(const PvIn& v, const StepRegs& s, float (&o)[8][2][4], float& u0,
                                        float& u1) {
    if (__any_sync(0xffffffffu, v.al0 != 1.f || v.al1 != 1.f)) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                o[ks][hf][0] *= v.al0; o[ks][hf][1] *= v.al0;
                o[ks][hf][2] *= v.al1; o[ks][hf][3] *= v.al1;
            }
        u0 *= v.al0;
        u1 *= v.al1;
    }
    u0 += v.p00.x * s.mu[0][0] + v.p00.y * s.mu[0][1] + v.p02.x * s.mu[1][0] + v.p02.y * s.mu[1][1];
    u1 += v.p10.x * s.mu[0][0] + v.p10.y * s.mu[0][1] + v.p12.x * s.mu[1][0] + v.p12.y * s.mu[1][1];
    uint32_t pa[4];
    pa[0] = pack_bf16(v.p00.x * s.sc[0][0], v.p00.y * s.sc[0][1]);
    pa[1] = pack_bf16(v.p10.x * s.sc[0][0], v.p10.y * s.sc[0][1]);
    pa[2] = pack_bf16(v.p02.x * s.sc[1][0], v.p02.y * s.sc[1][1]);
    pa[3] = pack_bf16(v.p12.x * s.sc[1][0], v.p12.y * s.sc[1][1]);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
            mma_bf16_16816(o[ks][hf], pa, movmatrix_trans(s.bq[0][ks][hf]), movmatrix_trans(s.bq[1][ks][hf]));
}

__global__ void __launch_bounds__(kDecodeThreads, 1)
rolaq_decode_split(const __grid_constant__ CUtensorMap map32, const __grid_constant__ CUtensorMap map8,
                   const DecodeArgs args) {
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
        for (int t = 0; t < 2; ++t)
            for (int s = 0; s < kNStage; ++s) mbar_init(smem_u32(&sm.full[t][s]), 1);
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map32);
        prefetch_tmap(&map8);
    }
    __syncthreads();
    const int b = sm.plan[0];
    if (b < 0) return;                         // item past the end of the plan
    const int first_page = sm.plan[1], n_pages = sm.plan[2];
    const int L = args.seq_lens[b];
    const int item = blockIdx.x;
    const int team = warp >> 2, g = warp & 3;
    const bool producer = (g == 0) && (lane == 0);
    if (producer)
        for (int k = 0; k < n_pages && k < kNStage; ++k)
            load_half_page(sm, &map32, &map8, args, team, b, first_page + k, k);

    const int r = lane >> 2, i = lane & 3;     // mma fragment row group / thread in group
    const int h0 = hc * 16;
    const __nv_bfloat16* qrow0 = args.q + ((size_t)b * args.heads + h0 + r) * ROLAQ_D_C + 128 * g;
    const __nv_bfloat16* qrow1 = qrow0 + 8 * ROLAQ_D_C;

    // Query fragments for this warp's group, in the qk_channel order; row sums of q_g.
    uint32_t qa[8][4];
    float qs0 = 0.f, qs1 = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const int c0 = qk_channel(s, 2 * i), c1 = qk_channel(s, 2 * i + 1);
        const int c2 = qk_channel(s, 2 * i + 8), c3 = qk_channel(s, 2 * i + 9);
        const float v00 = __bfloat162float(qrow0[c0]), v01 = __bfloat162float(qrow0[c1]);
        const float v02 = __bfloat162float(qrow0[c2]), v03 = __bfloat162float(qrow0[c3]);
        const float v10 = __bfloat162float(qrow1[c0]), v11 = __bfloat162float(qrow1[c1]);
        const float v12 = __bfloat162float(qrow1[c2]), v13 = __bfloat162float(qrow1[c3]);
        qa[s][0] = pack_bf16(v00, v01);
        qa[s][1] = pack_bf16(v10, v11);
        qa[s][2] = pack_bf16(v02, v03);
        qa[s][3] = pack_bf16(v12, v13);
        qs0 += (v00 + v01) + (v02 + v03);
        qs1 += (v10 + v11) + (v12 + v13);
    }
    qs0 += __shfl_xor_sync(0xffffffffu, qs0, 1);
    qs0 += __shfl_xor_sync(0xffffffffu, qs0, 2);
    qs1 += __shfl_xor_sync(0xffffffffu, qs1, 1);
    qs1 += __shfl_xor_sync(0xffffffffu, qs1, 2);
    uint32_t qra[4];
    {
        const uint32_t* r0 = reinterpret_cast<const uint32_t*>(
            args.qr + ((size_t)b * args.heads + h0 + r) * ROLAQ_D_R + 16 * g);
        const uint32_t* r1 = r0 + 8 * ROLAQ_D_R / 2;
        qra[0] = r0[i];
        qra[1] = r1[i];
        qra[2] = r0[4 + i];
        qra[3] = r1[4 + i];
    }

    float o[8][2][4];
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[s][hf][c] = 0.f;
    float u0 = 0.f, u1 = 0.f;                 // mean-term accumulators, rows r and r+8
    float m_ref = -INFINITY, l_part = 0.f;    // softmax state of head 4g + lane/8 (this lane's share)
    const int hh = 4 * g + (lane >> 3), jj = lane & 7;

    const uint32_t lut_lo = args.lut_lo, lut_hi = args.lut_hi;
    const bool protect = args.n_sink > 0 || args.n_recent > 0;
    const int recent_start = L - args.n_recent;
    const int bar_id = 1 + team;

    // QK of step (page k, sub) into regs: waits for the stage when sub == 0.
    auto qk = [&](int k, int sub, int buf, StepRegs& regs) {
        const int st = k % kNStage;
        if (sub == 0) mbar_wait(smem_u32(&sm.full[team][st]), (k / kNStage) & 1, &sm.abort);
        const int pos0 = (first_page + k) * kPageTok + 32 * team + kStepTok * sub;
        const int nvalid = sm.valid[team][st] ? min(max(L - pos0, 0), kStepTok) : 0;
        const bool mixed = protect && (pos0 < args.n_sink || pos0 + kStepTok > recent_start);
        if (nvalid == kStepTok && !mixed)
            qk_step<true>(sm.stage[team][st], sub, sm.sT[team][buf][g], r, i, g, lut_lo, lut_hi, args.kappa,
                          qa, qra, qs0, qs1, kStepTok, pos0, L, recent_start, args, b, regs);
        else
            qk_step<false>(sm.stage[team][st], sub, sm.sT[team][buf][g], r, i, g, lut_lo, lut_hi, args.kappa,
                           qa, qra, qs0, qs1, nvalid, pos0, L, recent_start, args, b, regs);
    };

    StepRegs ra, rb;
    if (n_pages > 0) {
        qk(0, 0, 0, ra);
        named_bar_sync(bar_id, 128);
        softmax_step(sm.sT[team][0], sm.sP[team][0], sm.sAl[team][0], hh, jj, args.scale_log2, m_ref, l_part);
    }
    for (int k = 0; k < n_pages; ++k) {
        // step 2k+1 (second 16 tokens of page k) into rb; PV of step 2k from ra
        qk(k, 1, 1, rb);
        named_bar_sync(bar_id, 128);
        // every warp of the team is done reading stage k: refill it
        if (producer && k + kNStage < n_pages)
            load_half_page(sm, &map32, &map8, args, team, b, first_page + k + kNStage, k + kNStage);
        const PvIn va = pv_load(sm.sP[team][0], sm.sAl[team][0], r, i);
        softmax_step(sm.sT[team][1], sm.sP[team][1], sm.sAl[team][1], hh, jj, args.scale_log2, m_ref, l_part);
        pv_step(va, ra, o, u0, u1);
        // step 2k+2 (first 16 tokens of page k+1) into ra; PV of step 2k+1 from rb
        const bool more = k + 1 < n_pages;
        if (more) qk(k + 1, 0, 0, ra);
        named_bar_sync(bar_id, 128);
        const PvIn vb = pv_load(sm.sP[team][1], sm.sAl[team][1], r, i);
        if (more)
            softmax_step(sm.sT[team][0], sm.sP[team][0], sm.sAl[team][0], hh, jj, args.scale_log2, m_ref, l_part);
        pv_step(vb, rb, o, u0, u1);
    }

    // ---- write this team's partial: O + mean term, and (m, l) per head ---------
    u0 += __shfl_xor_sync(0xffffffffu, u0, 1);
    u0 += __shfl_xor_sync(0xffffffffu, u0, 2);
    u1 += __shfl_xor_sync(0xffffffffu, u1, 1);
    u1 += __shfl_xor_sync(0xffffffffu, u1, 2);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 4);
    const size_t part = (size_t)item * 2 + team;
    float* out0 = args.ws_o + (part * args.heads + h0 + r) * ROLAQ_D_C + 128 * g;
    float* out1 = out0 + 8 * ROLAQ_D_C;
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int ch = 32 * i + 16 * (s >> 2) + 8 * hf + 4 * e + (s & 3);
                out0[ch] = o[s][hf][e] + u0;
                out1[ch] = o[s][hf][2 + e] + u1;
            }
    if (jj == 0) args.ws_ml[part * args.heads + h0 + hh] = make_float2(m_ref, l_part);
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
    const int p0 = 2 * s_plan[0], np = 2 * s_plan[1];
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
