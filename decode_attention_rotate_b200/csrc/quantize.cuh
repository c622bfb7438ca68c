// Write path ("RoLaQ", §3.2, §3.3, §A.3): y = c . R on the 5th-generation tensor cores,
// then per 128-coordinate group: mean, population std, four-level codes by tau, 2-bit
// packing, (mean, gain*std) metadata, the bf16 RoPE key copy and, for protected tokens,
// bf16(y) into the side store.
//
// rolaq_quantize_kernel is persistent (one CTA per SM).  A tile is 128 tokens (the TMEM
// lanes); its c block stays in shared memory while the four groups of 128 output
// coordinates are produced one after the other (one job per group); the tiles of a last,
// at most half-full round are split in two units of two groups.  Warp roles:
//   warp 8      producer: bulk tensor copies of the c tile (8 chunks of 128 x 64) and
//               of the R-plane chunks (128 x 64, 128-byte swizzle) each job needs;
//   warp 9      allocates 512 TMEM columns and issues tcgen05.mma (M=128, N=128, K=16,
//               bf16 in, fp32 accumulate).  R = R_hi + R_mid + R_lo (three bf16 planes,
//               ~2^-26 relative).  The tensor cores truncate each fp32 accumulation step
//               toward zero, so a job keeps two accumulators: chain A takes R_lo and R_mid
//               over all of K first (while it is small) and then R_hi over K < 256, chain B
//               takes R_hi over K >= 256; y = A + B.  That bounds the bias to 16 large
//               truncations per chain.  Jobs alternate between two TMEM buffers, so the
//               epilogue of one group overlaps the MMAs of the next;
//   warps 0..7  epilogue in two sets of four; set e quantizes groups e and e + 2.
#pragma once
#include "common.cuh"

namespace rolaq {

constexpr int kQTileM = 128;                  // tokens per tile (TMEM lanes)
constexpr int kQN = ROLAQ_GROUP;              // output coordinates per job: one group
constexpr int kQK = 64;                       // K per chunk (128-byte rows, 128B swizzle)
constexpr int kQKSteps = ROLAQ_D_C / kQK;     // 8
constexpr int kQStages = 3;
constexpr int kQThreads = 320;
constexpr int kQPlanes = 3;
constexpr uint32_t kQChunkBytes = kQTileM * kQK * 2;      // 16 KB (c chunk or one R-plane chunk)

struct QuantArgs {
    uint8_t* pages;
    int64_t num_pages;
    const int32_t* page_table;
    int max_pages, batch;
    __nv_bfloat16* prot;
    int n_sink, n_recent;
    const int32_t* req;
    const int32_t* pos;
    const int32_t* seq_lens;
    const __nv_bfloat16* k_r;   // [n][64]
    int n;
    float tau, gain;
};

struct QuantSmem {
    alignas(1024) uint8_t a[kQKSteps][kQChunkBytes];        // resident c tile, 8 K chunks
    alignas(1024) uint8_t b[kQStages][2][kQChunkBytes];     // streamed R-plane chunks
    alignas(8) uint64_t a_full[kQKSteps];
    uint64_t a_free[kQKSteps];
    uint64_t full[kQStages];
    uint64_t empty[kQStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(QuantSmem) + 1024 <= 227 * 1024, "write-path shared memory");

// Shared-memory matrix descriptor: K-major operand, 128-byte rows with 128B swizzle,
// 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    return smem_desc(saddr, 16, 1024, 2);
}
// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128, N = 128.
constexpr uint32_t kQIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kQN >> 3) << 17) |
                             ((uint32_t)(kQTileM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(da), "l"(db), "r"(kQIdesc), "r"(acc) : "memory");
}
// 16 columns of y = chain A + chain B (fp32 add of the two K-half accumulators).
__device__ __forceinline__ void load_y16(uint32_t col_a, uint32_t col_b, float (&y)[16]) {
    uint32_t ua[16], ub[16];
    tmem_ld16(col_a, ua);
    tmem_ld16(col_b, ub);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) y[j] = __uint_as_float(ua[j]) + __uint_as_float(ub[j]);
}

// Quantize one 128-coordinate group of one token straight from TMEM (this thread's lane;
// chain A at col_a.., chain B at col_b..), streaming 16 columns at a time in three
// passes: mean, population std, then codes (and the bf16 copy for a protected token).
// All lanes of the warp must call it (the TMEM loads are warp-wide); `store` is false for
// lanes without a valid target.
__device__ __forceinline__ void quantize_group_tmem(uint32_t col_a, uint32_t col_b, float tau, float gain,
                                                    bool store, uint8_t* dst_codes, float* dst_meta,
                                                    __nv_bfloat16* dst_prot) {
    float y[16];
    float s = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        load_y16(col_a + 16 * c, col_b + 16 * c, y);
#pragma unroll
        for (int j = 0; j < 16; ++j) s += y[j];
    }
    const float mean = s * (1.f / 128.f);
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        load_y16(col_a + 16 * c, col_b + 16 * c, y);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float d = y[j] - mean;
            ss = fmaf(d, d, ss);
        }
    }
    const float sd = sqrtf(ss * (1.f / 128.f));
    // z = (y - mean) / sd against -tau, 0, tau; a group with sd == 0 gets z = 0.
    const float inv = sd > 0.f ? 1.f / sd : 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
        load_y16(col_a + 16 * c, col_b + 16 * c, y);
        uint32_t acc = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float z = (y[j] - mean) * inv;
            const uint32_t code = (uint32_t)(z >= -tau) + (uint32_t)(z >= 0.f) + (uint32_t)(z >= tau);
            acc |= code << (2 * j);
        }
        if (store) reinterpret_cast<uint32_t*>(dst_codes)[c] = acc;      // 16 codes
        if (store && dst_prot) {
            uint4* dp = reinterpret_cast<uint4*>(dst_prot + 16 * c);
#pragma unroll
            for (int q8 = 0; q8 < 2; ++q8)
                dp[q8] = make_uint4(pack_bf16(y[8 * q8 + 0], y[8 * q8 + 1]), pack_bf16(y[8 * q8 + 2], y[8 * q8 + 3]),
                                    pack_bf16(y[8 * q8 + 4], y[8 * q8 + 5]), pack_bf16(y[8 * q8 + 6], y[8 * q8 + 7]));
        }
    }
    if (store) *reinterpret_cast<float2*>(dst_meta) = make_float2(mean, gain * sd);
}

// Work units of the persistent grid: CTA b takes tiles b, b + grid, ... whole (all four
// groups); when the last round is at most half full, each of its tiles is split in two
// units of two groups (groups 0-1 and 2-3 on CTAs 2j and 2j + 1), so that round costs
// half a tile.  Every role of a CTA walks the same units.
struct QUnit { int tile, g0, ng; };
__device__ __forceinline__ int q_unit_count(int n_tiles, int cta) {
    const int grid = (int)gridDim.x, full = n_tiles / grid, rem = n_tiles % grid;
    const bool split = rem > 0 && 2 * rem <= grid;
    return full + ((split ? cta < 2 * rem : cta < rem) ? 1 : 0);
}
__device__ __forceinline__ QUnit q_unit(int n_tiles, int cta, int k) {
    const int grid = (int)gridDim.x, full = n_tiles / grid, rem = n_tiles % grid;
    if (k < full) return QUnit{k * grid + cta, 0, ROLAQ_GROUPS};
    if (rem > 0 && 2 * rem <= grid) return QUnit{full * grid + cta / 2, 2 * (cta & 1), 2};
    return QUnit{full * grid + cta, 0, ROLAQ_GROUPS};
}

__global__ void __launch_bounds__(kQThreads, 1)
rolaq_quantize_kernel(const __grid_constant__ CUtensorMap map_c,
                      const __grid_constant__ CUtensorMap map_r, const QuantArgs args) {
    extern __shared__ uint8_t smem_raw[];
    // offset the __shared__ array itself (not an integer address) so that every access
    // stays a shared-memory access
    QuantSmem& sm = *reinterpret_cast<QuantSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (args.n + kQTileM - 1) / kQTileM;

    if (threadIdx.x == 0) {
        for (int k = 0; k < kQKSteps; ++k) {
            mbar_init(smem_u32(&sm.a_full[k]), 1);
            mbar_init(smem_u32(&sm.a_free[k]), 1);
        }
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&sm.tfull[a]), 1);
            mbar_init(smem_u32(&sm.tempty[a]), 4);
        }
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                     :: "r"(smem_u32(&sm.tmem_base)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 8 && lane == 0) { prefetch_tmap(&map_c); prefetch_tmap(&map_r); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    grid_dependency_wait();                    // launched as a dependent: inputs visible from here
    if (threadIdx.x == 0) grid_launch_dependents();

    if (warp == 8) {
        // ------------------------------------------------------------- producer --
        // Per tile: the 16 c chunks (once, kept for all four groups) and, per group, the
        // R_lo/R_mid chunks of the first pass then the R_hi chunks of the second.
        if (lane == 0) {
            uint32_t it = 0;
            int tl = 0;
            bool ok = true;
            const int nu = q_unit_count(n_tiles, (int)blockIdx.x);
            for (int un = 0; un < nu && ok; ++un, ++tl) {
                const QUnit w = q_unit(n_tiles, (int)blockIdx.x, un);
                const int tile = w.tile;
                for (int g = w.g0; g < w.g0 + w.ng && ok; ++g)
                    for (int pass = 0; pass < 2 && ok; ++pass)
                        for (int kc = 0; kc < kQKSteps; ++kc, ++it) {
                            if (g == w.g0 && pass == 0) {
                                if (tl > 0 && !mbar_wait(smem_u32(&sm.a_free[kc]), (tl - 1) & 1, &sm.abort)) {
                                    ok = false;
                                    break;
                                }
                                mbar_arrive_expect_tx(smem_u32(&sm.a_full[kc]), kQChunkBytes);
                                tma_load_2d(smem_u32(sm.a[kc]), &map_c, kc * kQK, tile * kQTileM,
                                            smem_u32(&sm.a_full[kc]));
                            }
                            const int st = it % kQStages;
                            if (it >= kQStages &&
                                !mbar_wait(smem_u32(&sm.empty[st]), ((it / kQStages) - 1) & 1, &sm.abort)) {
                                ok = false;
                                break;
                            }
                            const uint32_t fb = smem_u32(&sm.full[st]);
                            const int n0 = g * kQN;
                            if (pass == 0) {    // R_lo and R_mid (planes 2, 1)
                                mbar_arrive_expect_tx(fb, 2 * kQChunkBytes);
                                tma_load_2d(smem_u32(sm.b[st][0]), &map_r, kc * kQK, 2 * ROLAQ_D_C + n0, fb);
                                tma_load_2d(smem_u32(sm.b[st][1]), &map_r, kc * kQK, ROLAQ_D_C + n0, fb);
                            } else {            // R_hi (plane 0)
                                mbar_arrive_expect_tx(fb, kQChunkBytes);
                                tma_load_2d(smem_u32(sm.b[st][0]), &map_r, kc * kQK, n0, fb);
                            }
                        }
            }
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------------- MMA ----
        // Chain A (TMEM columns buf*256 .. +127): R_lo and R_mid over all of K, then R_hi
        // over K < 256.  Chain B (+128 .. +255): R_hi over K >= 256.  y = A + B.
        // The whole warp runs the loop (waits and descriptors are warp-uniform, so the
        // operands stay in uniform registers); one elected lane issues each chunk's MMAs
        // and commits.
        {
            uint32_t it = 0, job = 0;
            int tl = 0;
            bool ok = true;
            const int nu = q_unit_count(n_tiles, (int)blockIdx.x);
            for (int un = 0; un < nu && ok; ++un, ++tl) {
                const QUnit w = q_unit(n_tiles, (int)blockIdx.x, un);
                for (int g = w.g0; g < w.g0 + w.ng && ok; ++g, ++job) {
                    const uint32_t buf = job & 1, use = job >> 1;
                    if (use >= 1)
                        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.tempty[buf]), (use - 1) & 1, &sm.abort));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d_a = tmem + buf * 2 * kQN, d_b = d_a + kQN;
                    for (int pass = 0; pass < 2 && ok; ++pass)
                        for (int kc = 0; kc < kQKSteps; ++kc, ++it) {
                            if (g == w.g0 && pass == 0)
                                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.a_full[kc]), tl & 1, &sm.abort));
                            const int st = it % kQStages;
                            if (ok)
                                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full[st]), (it / kQStages) & 1, &sm.abort));
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t sa = smem_u32(sm.a[kc]);
                            const uint32_t sb0 = smem_u32(sm.b[st][0]), sb1 = smem_u32(sm.b[st][1]);
                            if (elect_one()) {
#pragma unroll
                                for (int k16 = 0; k16 < kQK / 16; ++k16) {
                                    const uint64_t da = umma_desc_sw128(sa + 32 * k16);
                                    const uint64_t db0 = umma_desc_sw128(sb0 + 32 * k16);
                                    if (pass == 0) {
                                        umma_bf16(d_a, da, db0, (kc | k16) != 0);
                                        umma_bf16(d_a, da, umma_desc_sw128(sb1 + 32 * k16), 1u);
                                    } else if (kc < kQKSteps / 2) {
                                        umma_bf16(d_a, da, db0, 1u);
                                    } else {
                                        umma_bf16(d_b, da, db0, (kc > kQKSteps / 2 || k16 > 0) ? 1u : 0u);
                                    }
                                }
                                umma_commit(smem_u32(&sm.empty[st]));
                                if (g == w.g0 + w.ng - 1 && pass == 1) umma_commit(smem_u32(&sm.a_free[kc]));
                            }
                            __syncwarp();
                        }
                    if (ok) {
                        if (elect_one()) umma_commit(smem_u32(&sm.tfull[buf]));
                        __syncwarp();
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue ----
        // Two sets of four warps take alternate groups (set e: groups e and e + 2, TMEM
        // buffer e); warp q of a set reads TMEM lanes 32q.. (one token per thread).
        const int q = warp & 3, set = warp >> 2;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t use = 0;
        const int nu = q_unit_count(n_tiles, (int)blockIdx.x);
        for (int un = 0; un < nu; ++un) {
            const QUnit w = q_unit(n_tiles, (int)blockIdx.x, un);
            // Target slot of this thread's token, looked up before the accumulator is ready
            // so the dependent global loads overlap the MMAs.
            const int tok = w.tile * kQTileM + 32 * q + lane;
            long long pid = -1;
            int rq = -1, ps = 0;
            if (tok < args.n) {
                rq = args.req[tok];
                ps = args.pos[tok];
                if (rq >= 0 && rq < args.batch && ps >= 0 && (ps / ROLAQ_PAGE_TOKENS) < args.max_pages) {
                    pid = args.page_table[(long long)rq * args.max_pages + ps / ROLAQ_PAGE_TOKENS];
                    if (pid >= args.num_pages) pid = -1;
                }
                if (pid < 0 && set == 0) raise_status(ROLAQ_STATUS_BAD_SLOT);
            }
            const bool store = pid >= 0;
            uint8_t* page = args.pages + (store ? pid : 0) * (long long)ROLAQ_PAGE_BYTES;
            const int row = ps % ROLAQ_PAGE_TOKENS;
            long long prot_row = -1;                  // side-store row of a protected token
            if (store && args.prot) {
                const int nslot = args.n_sink + args.n_recent;
                if (ps < args.n_sink)
                    prot_row = (long long)rq * nslot + ps;
                else if (args.n_recent > 0 && ps >= args.seq_lens[rq] - args.n_recent)
                    prot_row = (long long)rq * nslot + args.n_sink + ps % args.n_recent;
            }
            if (store && set == 0 && w.g0 == 0) {
                const uint4* src = reinterpret_cast<const uint4*>(args.k_r + (size_t)tok * ROLAQ_D_R);
                uint4* dst = reinterpret_cast<uint4*>(page + ROLAQ_PAGE_KR_OFFSET + row * ROLAQ_KR_BYTES);
#pragma unroll
                for (int j = 0; j < 8; ++j) dst[j] = src[j];
            }
            for (int g = w.g0 + set; g < w.g0 + w.ng; g += 2, ++use) {
                const bool got = mbar_wait(smem_u32(&sm.tfull[set]), use & 1, &sm.abort);
                tc_fence_after();
                __nv_bfloat16* prot = prot_row >= 0 ? args.prot + prot_row * ROLAQ_D_C + 128 * g : nullptr;
                const uint32_t col = tmem + lane_base + (uint32_t)(set * 2 * kQN);
                quantize_group_tmem(col, col + kQN, args.tau, args.gain, store && got,
                                    page + ROLAQ_PAGE_CODES_OFFSET + row * ROLAQ_CODE_BYTES + 32 * g,
                                    reinterpret_cast<float*>(page + ROLAQ_PAGE_META_OFFSET + row * ROLAQ_META_BYTES) + 2 * g,
                                    prot);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.tempty[set]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" :: "r"(tmem) : "memory");
    }
}

// R (fp32 [512 in][512 out], y = c . R) -> three bf16 planes [3][512 out][512 in]: the
// nearest bf16 of R^T, of the remainder, and of what remains after that.
__global__ void rolaq_split_rotation(const float* __restrict__ R, __nv_bfloat16* __restrict__ out) {
    const int o = blockIdx.x;                  // output coordinate (row of R^T)
    const size_t plane = (size_t)ROLAQ_D_C * ROLAQ_D_C;
    for (int k = threadIdx.x; k < ROLAQ_D_C; k += blockDim.x) {
        const float x = R[(size_t)k * ROLAQ_D_C + o];
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        out[(size_t)o * ROLAQ_D_C + k] = hi;
        out[plane + (size_t)o * ROLAQ_D_C + k] = mid;
        out[2 * plane + (size_t)o * ROLAQ_D_C + k] = lo;
    }
}

}  // namespace rolaq

namespace rolaq {

// ---- small appends --------------------------------------------------------------
// A decode step appends one token per request: a few tokens per call.  The tensor-core
// kernel above would stream all of R through a single CTA for them, so small calls use
// this kernel instead: a cluster of kSmallSlices CTAs per (group, 8 tokens), so that the
// group's 384 KB of R-plane rows are read by eight SMs.  CTA s of a cluster computes
// output coordinates 128g + 16s .. +15, two per warp: for each, the 32 lanes read the
// three R-plane rows coalesced (16 inputs each), sum the planes in fp32 (smallest first),
// multiply-add the CTA's tokens and reduce across the warp; the results go straight into
// the shared memory of the cluster's first CTA, which computes the group statistics
// (block reductions) and stores the records.
constexpr int kSmallTok = 8;
constexpr int kSmallMaxN = 64;
constexpr int kSmallSlices = 8;
constexpr int kSmallThreads = 256;
constexpr int kSmallOutPerCta = ROLAQ_GROUP / kSmallSlices;                  // 16
constexpr int kSmallOutPerWarp = kSmallOutPerCta / (kSmallThreads / 32);    // 2

__device__ __forceinline__ float block_sum128(float v, float* red) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const float r = (red[0] + red[1]) + (red[2] + red[3]);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    return r;
}

__global__ void __cluster_dims__(kSmallSlices, 1, 1) __launch_bounds__(kSmallThreads)
rolaq_quantize_small_kernel(const __nv_bfloat16* __restrict__ R_split, const __nv_bfloat16* __restrict__ c,
                            const QuantArgs args) {
    __shared__ __align__(16) __nv_bfloat16 s_c[kSmallTok][ROLAQ_D_C];
    __shared__ float s_y[kSmallTok][ROLAQ_GROUP];
    __shared__ float s_red[4];
    __shared__ uint32_t s_codes[kSmallTok][8];
    // each token's target, looked up before the dot products so that the dependent
    // global loads (request, position, page table, length) overlap them
    __shared__ long long s_pid[kSmallTok], s_prow[kSmallTok];
    __shared__ int s_row[kSmallTok];
    __shared__ __align__(16) uint2 s_kr[kSmallTok][ROLAQ_KR_BYTES / 8];
    const uint32_t rank = cluster_ctarank();     // output slice of the group
    const int g = blockIdx.y;                    // group
    const int t0 = blockIdx.z * kSmallTok;
    const int nt = min(kSmallTok, args.n - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < kSmallTok * ROLAQ_D_C / 8; e += blockDim.x) {
        const int t = e / (ROLAQ_D_C / 8), k8 = e % (ROLAQ_D_C / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < nt) v = reinterpret_cast<const uint4*>(c + (size_t)(t0 + t) * ROLAQ_D_C)[k8];
        reinterpret_cast<uint4*>(s_c[t])[k8] = v;
    }
    if (threadIdx.x < kSmallTok * 8) s_codes[threadIdx.x >> 3][threadIdx.x & 7] = 0;
    if (rank == 0 && threadIdx.x < nt) {
        const int t = threadIdx.x, tok = t0 + t;
        const int rq = args.req[tok], ps = args.pos[tok];
        long long pid = -1, prow = -1;
        if (rq >= 0 && rq < args.batch && ps >= 0 && (ps / ROLAQ_PAGE_TOKENS) < args.max_pages) {
            pid = args.page_table[(long long)rq * args.max_pages + ps / ROLAQ_PAGE_TOKENS];
            if (pid >= args.num_pages) pid = -1;
        }
        if (pid >= 0 && args.prot) {
            const int nslot = args.n_sink + args.n_recent;
            if (ps < args.n_sink)
                prow = (long long)rq * nslot + ps;
            else if (args.n_recent > 0 && ps >= args.seq_lens[rq] - args.n_recent)
                prow = (long long)rq * nslot + args.n_sink + ps % args.n_recent;
        }
        s_pid[t] = pid;
        s_prow[t] = prow;
        s_row[t] = ps % ROLAQ_PAGE_TOKENS;
    }
    if (rank == 0 && g == 0 && threadIdx.x >= 128 && threadIdx.x < 128 + kSmallTok * 16) {
        const int t = (threadIdx.x - 128) >> 4, j = threadIdx.x & 15;
        if (t < nt) s_kr[t][j] = reinterpret_cast<const uint2*>(args.k_r + (size_t)(t0 + t) * ROLAQ_D_R)[j];
    }
    __syncthreads();
    cluster_sync();                              // every CTA of the cluster is running
    const uint32_t y_first = mapa_shared(smem_u32(&s_y[0][0]), 0);
    const size_t plane = (size_t)ROLAQ_D_C * ROLAQ_D_C;
#pragma unroll
    for (int oo = 0; oo < kSmallOutPerWarp; ++oo) {
        const int o = kSmallOutPerCta * (int)rank + kSmallOutPerWarp * warp + oo;
        float rk[16];
#pragma unroll
        for (int q8 = 0; q8 < 16; ++q8) rk[q8] = 0.f;
#pragma unroll
        for (int pl = 2; pl >= 0; --pl) {        // smallest plane first
            const uint4* row = reinterpret_cast<const uint4*>(R_split + pl * plane + (size_t)(128 * g + o) * ROLAQ_D_C);
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
#pragma unroll
        for (int t = 0; t < kSmallTok; ++t) {
            float acc = 0.f;
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                const uint4 cu = reinterpret_cast<const uint4*>(s_c[t])[2 * lane + hv];
                const uint32_t cw[4] = {cu.x, cu.y, cu.z, cu.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc = fmaf(__uint_as_float(cw[q] << 16), rk[8 * hv + 2 * q], acc);
                    acc = fmaf(__uint_as_float(cw[q] & 0xFFFF0000u), rk[8 * hv + 2 * q + 1], acc);
                }
            }
            for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) st_cluster_f32(y_first + (uint32_t)(t * ROLAQ_GROUP + o) * 4u, acc);
        }
    }
    cluster_sync();                              // the group's y is complete in the first CTA
    if (rank != 0) return;
    if (threadIdx.x >= ROLAQ_GROUP) return;      // warps 0..3 finish the group
    const int j = threadIdx.x;
    for (int t = 0; t < nt; ++t) {
        const float y = s_y[t][j];
        const float mean = block_sum128(y, s_red) * (1.f / 128.f);
        const float d = y - mean;
        const float sd = sqrtf(block_sum128(d * d, s_red) * (1.f / 128.f));
        const float inv = sd > 0.f ? 1.f / sd : 0.f;
        const float z = d * inv;
        const uint32_t code = (uint32_t)(z >= -args.tau) + (uint32_t)(z >= 0.f) + (uint32_t)(z >= args.tau);
        atomicOr(&s_codes[t][j >> 4], code << (2 * (j & 15)));
        const long long pid = s_pid[t];
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (pid < 0) {
            if (j == 0 && g == 0) raise_status(ROLAQ_STATUS_BAD_SLOT);
            continue;
        }
        uint8_t* page = args.pages + pid * (long long)ROLAQ_PAGE_BYTES;
        const int row = s_row[t];
        if (j < 8)
            reinterpret_cast<uint32_t*>(page + ROLAQ_PAGE_CODES_OFFSET + row * ROLAQ_CODE_BYTES + 32 * g)[j] = s_codes[t][j];
        if (j == 0)
            *reinterpret_cast<float2*>(page + ROLAQ_PAGE_META_OFFSET + row * ROLAQ_META_BYTES + 8 * g) =
                make_float2(mean, args.gain * sd);
        if (g == 0 && j < 16) reinterpret_cast<uint2*>(page + ROLAQ_PAGE_KR_OFFSET + row * ROLAQ_KR_BYTES)[j] = s_kr[t][j];
        const long long prow = s_prow[t];
        if (prow >= 0) args.prot[prow * ROLAQ_D_C + 128 * g + j] = __float2bfloat16_rn(y);
    }
}

}  // namespace rolaq
