// Decode with quantisation disabled: every token protected, so x is the bf16 side-store row
// of each token ("RoLaQ", §4.1 "Setup", §A.3: protected tokens keep BF16 content) and the
// RoPE key comes from the page.  This is the BF16 MLA decode on the same cache layout.
//
// rolaq_decode_bf16<HC>: one CTA per (work item, chunk of HC = 16 or 32 heads), the split
// plan of the 2-bit decode, 8 warps.  Per 64-token page:
//   warp 0 (lane 0)   copies the page's 64 side-store rows as eight 64 x 64 bf16 boxes with
//                     the 128-byte swizzle (which is the x-tile layout the tensor cores
//                     read, so no dequantisation is needed) plus the page's 64 RoPE rows,
//                     into one of two stages;
//   warp 1            QK: tcgen05.mma M = 64 tokens, N = HC, K = 512 with A = the x tile
//                     (K-major, shared memory), B = the bf16 query, plus K = 64 RoPE; on the
//                     request's last page it first zeroes the tile rows past the sequence
//                     end (the side store there holds no token);
//   warp 2            PV: M = 128 channels, K = 64 tokens, A = the same tile read MN-major,
//                     B = P in bf16 (an MMA takes one type for both operands);
//   warps 4..7        the softmax of the 2-bit decode (softmax_role), P in bf16.
// The channel order is the natural one (no lookup slots).  The merge kernel is shared.
#pragma once
#include "decode.cuh"

namespace rolaq {

constexpr int kBf16Threads = 256;
constexpr int kBStages = 2;
constexpr int kKrTile = kPageTok * 128;             // 64 RoPE rows of 128 B
constexpr int kBf16TmemCols = 256;

template <int HC>
struct Bf16Smem {
    alignas(1024) uint8_t x[kBStages][kXTile];          // bf16 x tiles (K-major, 128-byte swizzle)
    alignas(1024) uint8_t kr[kBStages][kKrTile];        // RoPE key rows (K-major, 128-byte swizzle)
    alignas(128) uint8_t qc[HC * ROLAQ_D_C * 2];        // bf16 query, QK B operand
    alignas(128) uint8_t qr[HC * ROLAQ_D_R * 2];        // bf16 RoPE query
    alignas(128) uint8_t P[kPBufs][HC * kPageTok * 2];  // bf16 probabilities, PV B operand
    float red[4][HC];
    float mref[HC];
    float alpha[HC];
    alignas(8) uint64_t full[kBStages];    // x tile and RoPE rows landed
    alignas(8) uint64_t xfree[kBStages];   // PV of the stage done (QK of it done earlier)
    alignas(8) uint64_t sfull[2];
    alignas(8) uint64_t sfree[2];
    alignas(8) uint64_t pready[kPBufs];
    alignas(8) uint64_t pdone[kPBufs];
    uint32_t tmem_base;
    int plan[4];
    int abort;
};
static_assert(sizeof(Bf16Smem<16>) + 1024 <= 227 * 1024, "bf16 decode shared memory (16 heads)");
static_assert(sizeof(Bf16Smem<32>) + 1024 <= 227 * 1024, "bf16 decode shared memory (32 heads)");

// Side-store slot of position p (all positions of a page share one contiguous run when
// n_sink and n_recent are multiples of 64).
__device__ __forceinline__ int prot_slot(const DecodeArgs& args, int p) {
    if (p < args.n_sink || args.n_recent == 0) return p;
    return args.n_sink + p % args.n_recent;
}

template <int HC>
__global__ void __launch_bounds__(kBf16Threads, 1)
rolaq_decode_bf16(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_kr,
                  const DecodeArgs args) {
    extern __shared__ uint8_t smem_raw[];
    constexpr uint32_t kIdQk = id_rope<HC>();                                // bf16 x bf16, M = 64
    constexpr uint32_t kIdPv = id_pv<HC>() | (1u << 7) | (1u << 10);         // bf16, M = 128, A MN-major
    static_assert(kOCol + 4 * HC <= kBf16TmemCols && kSCol + 2 * HC <= kOCol, "tensor-memory columns");
    Bf16Smem<HC>& sm =
        *reinterpret_cast<Bf16Smem<HC>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h0 = blockIdx.y * HC;
    grid_dependency_wait();                    // the previous kernel's output is visible from here

    if (warp == 0) {
        PlanInfo pi = plan_lookup(args.seq_lens, args.batch, args.target_items, (int)blockIdx.x, -1, 0);
        if (lane == 0) {
            sm.plan[0] = pi.b;
            sm.plan[1] = pi.first_page;
            sm.plan[2] = pi.n_pages;
        }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.xfree[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&sm.sfull[s]), 1);
            mbar_init(smem_u32(&sm.sfree[s]), 4);
        }
        for (int s = 0; s < kPBufs; ++s) {
            mbar_init(smem_u32(&sm.pready[s]), 4);
            mbar_init(smem_u32(&sm.pdone[s]), 1);
        }
        for (int h = 0; h < HC; ++h) sm.mref[h] = -INFINITY;
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_x);
        prefetch_tmap(&map_kr);
    }
    __syncthreads();
    const int b = sm.plan[0];
    if (b < 0) return;                         // item past the end of the plan
    const int first_page = sm.plan[1], T = sm.plan[2];
    const int L = args.seq_lens[b];
    // a position outside the sink and recent windows has no bf16 copy
    if (threadIdx.x == 0 && blockIdx.y == 0 && L - args.n_recent > args.n_sink) raise_status(ROLAQ_STATUS_BAD_SLOT);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&sm.tmem_base)), "r"(kBf16TmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // queries as B operands, bf16, channel order
    {
        const uint32_t* qb = reinterpret_cast<const uint32_t*>(args.q + ((size_t)b * args.heads + h0) * ROLAQ_D_C);
        for (int e = threadIdx.x; e < HC * ROLAQ_D_C / 2; e += kBf16Threads) {
            const int n = e / (ROLAQ_D_C / 2), k = 2 * (e % (ROLAQ_D_C / 2));
            *reinterpret_cast<uint32_t*>(sm.qc + plain_off(n, k, 64 * 128)) = qb[e];
        }
        const uint32_t* rb = reinterpret_cast<const uint32_t*>(args.qr + ((size_t)b * args.heads + h0) * ROLAQ_D_R);
        for (int e = threadIdx.x; e < HC * ROLAQ_D_R / 2; e += kBf16Threads) {
            const int n = e / (ROLAQ_D_R / 2), k = 2 * (e % (ROLAQ_D_R / 2));
            *reinterpret_cast<uint32_t*>(sm.qr + plain_off(n, k, 8 * 128)) = rb[e];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int nslot = args.n_sink + args.n_recent;
    if (threadIdx.x == 0) grid_launch_dependents();     // the merge may be scheduled as CTAs finish

    if (warp == 0) {
        // ------------------------------------------------------------ producer ----
        if (lane == 0)
            for (int k = 0; k < T; ++k) {
                const int st = k % kBStages;
                if (k >= kBStages)
                    mbar_wait(smem_u32(&sm.xfree[st]), (unsigned)((k / kBStages - 1) & 1), &sm.abort);
                const int page = first_page + k;
                const long long pid = page_id(args, b, page);
                const bool ok = page_ok(args, pid);
                if (!ok) raise_status(ROLAQ_STATUS_BAD_PAGE);
                const uint32_t bar = smem_u32(&sm.full[st]);
                mbar_arrive_expect_tx(bar, kXTile + (ok ? kKrTile : 0));
                const int row0 = b * nslot + prot_slot(args, page * kPageTok);
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb)
                    tma_load_2d(smem_u32(sm.x[st]) + cb * kXAtom, &map_x, 64 * cb, row0, bar);
                if (ok) tma_load_2d(smem_u32(sm.kr[st]), &map_kr, 0, (int)(pid * kPageRows) + kKrRow, bar);
            }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- QK issue ----
        const uint64_t dqc = smem_desc(smem_u32(sm.qc), 128, 64 * 128, 0);
        const uint64_t dqr = smem_desc(smem_u32(sm.qr), 128, 8 * 128, 0);
        const uint64_t dx = smem_desc(smem_u32(sm.x[0]), 16, 1024, 2);
        const uint64_t dkr = smem_desc(smem_u32(sm.kr[0]), 16, 1024, 2);
        for (int i = 0; i < T; ++i) {
            const int bi = i & 1, st = i % kBStages;
            if (i >= 2) mbar_wait(smem_u32(&sm.sfree[bi]), (unsigned)(((i - 2) >> 1) & 1), &sm.abort);
            mbar_wait(smem_u32(&sm.full[st]), (unsigned)((i / kBStages) & 1), &sm.abort);
            // rows past the sequence end: zero, so that their (masked) probabilities meet
            // finite values in PV
            const int rows_valid = L - (first_page + i) * kPageTok;
            if (rows_valid < kPageTok) {
                const int r0 = rows_valid > 0 ? rows_valid : 0;
                for (int e = r0 * 64 + lane; e < kPageTok * 64; e += 32) {      // 16-byte chunks
                    const int r = e >> 6, c = e & 63;                           // row, chunk
                    *reinterpret_cast<uint4*>(sm.x[st] + (c >> 3) * kXAtom + r * 128 + ((c & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            tc_fence_after();
            const uint32_t d = tmem + kSCol + HC * bi;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < ROLAQ_D_C / 16; ++kk)
                    umma_ss1(d, dx + (uint64_t)((st * kXTile + (kk >> 2) * kXAtom + (kk & 3) * 32) >> 4),
                             dqc + (uint64_t)((kk * 256) >> 4), kIdQk, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < ROLAQ_D_R / 16; ++kk)
                    umma_ss1(d, dkr + (uint64_t)((st * kKrTile + kk * 32) >> 4), dqr + (uint64_t)((kk * 256) >> 4),
                             kIdQk, 1u);
                umma_commit(smem_u32(&sm.sfull[bi]));
            }
            __syncwarp();
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------- PV issue ----
        const uint64_t dxm = smem_desc(smem_u32(sm.x[0]), kXAtom, 1024, 2);
        const uint64_t dp = smem_desc(smem_u32(sm.P[0]), 128, 1024, 0);
        for (int j = 0; j < T; ++j) {
            const int st = j % kBStages, pj = j % kPBufs;
            mbar_wait(smem_u32(&sm.pready[pj]), (unsigned)((j / kPBufs) & 1), &sm.abort);
            __syncwarp();
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int ks = 0; ks < kPageTok / 16; ++ks)
                        umma_ss1(tmem + kOCol + HC * g,
                                 dxm + (uint64_t)((st * kXTile + 2 * g * kXAtom + ks * 2048) >> 4),
                                 dp + (uint64_t)((pj * (int)sizeof(sm.P[0]) + ks * 256) >> 4), kIdPv,
                                 (ks > 0 || j > 0) ? 1u : 0u);
                umma_commit(smem_u32(&sm.xfree[st]));
                umma_commit(smem_u32(&sm.pdone[pj]));
            }
            __syncwarp();
        }
    } else if (warp >= kSoftWarp0) {
        // ------------------------------------------------------------- softmax ----
        softmax_role<HC, true, false>(sm, args, tmem, warp, lane, b, first_page, T, L, h0, [&](int j) {
            mbar_wait(smem_u32(&sm.xfree[j % kBStages]), (unsigned)((j / kBStages) & 1), &sm.abort);
        });
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kBf16TmemCols)
                     : "memory");
    }
}

}  // namespace rolaq
