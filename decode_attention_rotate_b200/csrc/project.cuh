// Absorbed projections around the cache ("RoLaQ", §3.3; Fig. 3a): the read-side rotation
// folds into the query projection and its inverse into the value projection.
//   W_q[h] = W_UK[h]^T . R     [128][512]   (once per layer)
//   W_o[h] = R^T . W_UV[h]     [512][128]   (once per layer)
//   q_c_rot[b,h] = q_nope[b,h] . W_q[h]     (per decode step, bf16 out)
//   v[b,h]       = out_rot[b,h] . W_o[h]    (per decode step, fp32 out)
// The folded weights are stored in bf16 (the precision the model's own projections carry);
// every sum runs in fp32.
#pragma once
#include "common.cuh"

namespace rolaq {

// ---- once per layer: the weight fold (plain fp32 dot products, bf16 result) ---------

constexpr int kFoldThreads = 128;

// W_q[h][n][j] = sum_k W_UK[h][k][n] R[k][j]: grid (512 / 128, 128, heads), thread = j.
__global__ void __launch_bounds__(kFoldThreads)
rolaq_fold_wq(const float* __restrict__ W_UK, const float* __restrict__ R, __nv_bfloat16* __restrict__ W_q) {
    const int j = blockIdx.x * kFoldThreads + threadIdx.x, n = blockIdx.y, h = blockIdx.z;
    const float* wk = W_UK + (size_t)h * ROLAQ_D_C * ROLAQ_D_NOPE + n;
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < ROLAQ_D_C; ++k) acc = fmaf(wk[(size_t)k * ROLAQ_D_NOPE], R[(size_t)k * ROLAQ_D_C + j], acc);
    W_q[((size_t)h * ROLAQ_D_NOPE + n) * ROLAQ_D_C + j] = __float2bfloat16_rn(acc);
}

// W_o[h][k][n] = sum_j R[j][k] W_UV[h][j][n]: grid (512, heads), thread = n.
__global__ void __launch_bounds__(kFoldThreads)
rolaq_fold_wo(const float* __restrict__ W_UV, const float* __restrict__ R, __nv_bfloat16* __restrict__ W_o) {
    const int n = threadIdx.x, k = blockIdx.x, h = blockIdx.y;
    const float* wv = W_UV + (size_t)h * ROLAQ_D_C * ROLAQ_D_V + n;
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < ROLAQ_D_C; ++j) acc = fmaf(R[(size_t)j * ROLAQ_D_C + k], wv[(size_t)j * ROLAQ_D_V], acc);
    W_o[((size_t)h * ROLAQ_D_C + k) * ROLAQ_D_V + n] = __float2bfloat16_rn(acc);
}

// ---- per step: query fold and output unfold on the tensor cores ---------------------
// Both are D[m][b] = sum_k A[m][k] B[b][k] for one head:
//   fold:   m = 128 output columns j of a 128-column tile, k = n (K = 128), A = W_q[h]^T,
//           B = q_nope[., h]
//   unfold: m = the 128 value columns n, k = latent channel (K = 512), A = W_o[h]^T,
//           B = out[., h] rounded to bf16
// A is the folded weight read MN-major straight from its row-major layout: a bulk tensor
// copy of {64 columns x 128 rows} with 128-byte swizzle per block.  B holds up to kPjN
// queries, K-major in the no-swizzle core-matrix layout (8 rows x 16 bytes per core
// matrix), written by the CTA's threads; rows past the batch are zero.  One elected lane
// issues tcgen05.mma (M = 128, N = the queries rounded up to 16, fp32 accumulate in tensor
// memory) and each of the four warps reads its 32 tensor-memory lanes (32 output rows)
// in the epilogue.  The weights cross HBM once per call; the MMAs take well under a
// microsecond, so the kernels run at the weights' read time.

constexpr int kPjThreads = 128;
constexpr int kPjN = 64;                            // queries per MMA chunk (tensor-memory columns)
constexpr int kPjBlock = 128 * 128;                 // one {64 columns x 128 rows} bf16 block (16 KB)
constexpr int kPjStage = 8;                         // 16-byte chunks a thread loads before storing
// bf16 A and B, fp32 D, A MN-major, M = 128; N is or-ed in per chunk
constexpr uint32_t kIdProj = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((128u >> 4) << 24);

__device__ __forceinline__ uint32_t proj_idesc(int npad) { return kIdProj | ((uint32_t)(npad >> 3) << 17); }

struct FoldQSmem {
    alignas(1024) uint8_t a[2][kPjBlock];               // W_q tile: columns j0..j0+63, j0+64..j0+127
    alignas(128) uint8_t b[kPjN / 8][ROLAQ_D_NOPE / 8][128];   // queries: core matrices
    alignas(8) uint64_t full;
    alignas(8) uint64_t mma;
    uint32_t tmem;
    int abort;
};

struct UnfoldSmem {
    alignas(1024) uint8_t a[ROLAQ_D_C / 128][2][kPjBlock];     // W_o: 4 row chunks x 2 column blocks
    alignas(128) uint8_t b[kPjN / 8][ROLAQ_D_C / 8][128];     // outputs as bf16: core matrices
    alignas(8) uint64_t full[ROLAQ_D_C / 128];
    alignas(8) uint64_t mma;
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ void proj_tmem_alloc(uint32_t* slot) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(slot)), "r"(kPjN) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void proj_tmem_free(uint32_t tmem) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kPjN) : "memory");
}

// Epilogue: thread (warp w, lane l) owns output row m = 32w + l; columns are queries.
template <typename Store>
__device__ __forceinline__ void proj_epilogue(uint32_t tmem, int warp, int npad, Store store) {
    for (int c0 = 0; c0 < npad; c0 += 16) {
        uint32_t u[16];
        tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, u);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) store(c0 + i, __uint_as_float(u[i]));
    }
}

// grid (512 / 128 column tiles, heads), kPjThreads threads.
__global__ void __launch_bounds__(kPjThreads)
rolaq_fold_query_kernel(const __grid_constant__ CUtensorMap map_wq, const __nv_bfloat16* __restrict__ q_nope,
                        int batch, int heads, __nv_bfloat16* __restrict__ q_c_rot) {
    extern __shared__ uint8_t smem_raw[];
    FoldQSmem& sm = *reinterpret_cast<FoldQSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jt = blockIdx.x, h = blockIdx.y;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.full), 1);
        mbar_init(smem_u32(&sm.mma), 1);
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_wq);
    }
    if (warp == 0) proj_tmem_alloc(&sm.tmem);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    grid_dependency_wait();                    // launched as a dependent: inputs visible from here
    if (threadIdx.x == 0) grid_launch_dependents();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(smem_u32(&sm.full), 2 * kPjBlock);
        for (int c = 0; c < 2; ++c)
            tma_load_2d(smem_u32(sm.a[c]), &map_wq, jt * 128 + 64 * c, h * ROLAQ_D_NOPE, smem_u32(&sm.full));
    }
    const int m = 32 * warp + lane;
    for (int b0 = 0, it = 0; b0 < batch; b0 += kPjN, ++it) {
        const int nb = min(kPjN, batch - b0);
        const int npad = (nb + 15) & ~15;
        // npad x 16 chunks of 16 bytes: a multiple of the thread count; all of a thread's
        // loads are issued before its first store
        constexpr int kCpr = ROLAQ_D_NOPE / 8;
        for (int e0 = threadIdx.x; e0 < npad * kCpr; e0 += kPjStage * kPjThreads) {
            uint4 val[kPjStage];
#pragma unroll
            for (int u = 0; u < kPjStage; ++u) {
                const int e = e0 + u * kPjThreads, b = e / kCpr, c = e % kCpr;
                val[u] = make_uint4(0u, 0u, 0u, 0u);
                if (b < nb)
                    val[u] = *reinterpret_cast<const uint4*>(q_nope + ((size_t)(b0 + b) * heads + h) * ROLAQ_D_NOPE + 8 * c);
            }
#pragma unroll
            for (int u = 0; u < kPjStage; ++u) {
                const int e = e0 + u * kPjThreads, b = e / kCpr, c = e % kCpr;
                if (b < npad) *reinterpret_cast<uint4*>(&sm.b[b >> 3][c][(b & 7) * 16]) = val[u];
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (warp == 0) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full), 0, &sm.abort));
            if (ok) {
                tc_fence_after();
                const uint32_t idesc = proj_idesc(npad);
                const uint64_t da = smem_desc(smem_u32(sm.a[0]), kPjBlock, 1024, 2);
                const uint64_t db = smem_desc(smem_u32(&sm.b[0][0][0]), 128, (ROLAQ_D_NOPE / 8) * 128, 0);
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < ROLAQ_D_NOPE / 16; ++ks)
                        umma_ss1(tmem, da + (uint64_t)((ks * 2048) >> 4), db + (uint64_t)((ks * 256) >> 4), idesc,
                                 ks > 0 ? 1u : 0u);
                    umma_commit(smem_u32(&sm.mma));
                }
                __syncwarp();
            }
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.mma), (unsigned)(it & 1), &sm.abort));
        tc_fence_after();
        if (ok) {
            __nv_bfloat16* dst = q_c_rot + (size_t)h * ROLAQ_D_C + jt * 128 + m;
            proj_epilogue(tmem, warp, npad, [&](int b, float x) {
                if (b < nb) dst[(size_t)(b0 + b) * heads * ROLAQ_D_C] = __float2bfloat16_rn(x);
            });
        }
        tc_fence_before();
        __syncthreads();
        if (sm.abort) break;
    }
    tc_fence_after();
    if (warp == 0) proj_tmem_free(tmem);
}

// grid (heads), kPjThreads threads.
__global__ void __launch_bounds__(kPjThreads)
rolaq_unfold_output_kernel(const __grid_constant__ CUtensorMap map_wo, const float* __restrict__ out, int batch,
                           int heads, float* __restrict__ v) {
    extern __shared__ uint8_t smem_raw[];
    UnfoldSmem& sm = *reinterpret_cast<UnfoldSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    constexpr int kChunks = ROLAQ_D_C / 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x;
    if (threadIdx.x == 0) {
        for (int c = 0; c < kChunks; ++c) mbar_init(smem_u32(&sm.full[c]), 1);
        mbar_init(smem_u32(&sm.mma), 1);
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&map_wo);
    }
    if (warp == 0) proj_tmem_alloc(&sm.tmem);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    grid_dependency_wait();                    // launched as a dependent: inputs visible from here
    if (threadIdx.x == 0) grid_launch_dependents();
    if (threadIdx.x == 0) {
        for (int kc = 0; kc < kChunks; ++kc) {
            mbar_arrive_expect_tx(smem_u32(&sm.full[kc]), 2 * kPjBlock);
            for (int c = 0; c < 2; ++c)
                tma_load_2d(smem_u32(sm.a[kc][c]), &map_wo, 64 * c, h * ROLAQ_D_C + 128 * kc, smem_u32(&sm.full[kc]));
        }
    }
    const int m = 32 * warp + lane;
    for (int b0 = 0, it = 0; b0 < batch; b0 += kPjN, ++it) {
        const int nb = min(kPjN, batch - b0);
        const int npad = (nb + 15) & ~15;
        // npad x 64 chunks of 8 channels; all of a thread's loads are issued before its
        // first store
        constexpr int kCpr = ROLAQ_D_C / 8;
        for (int e0 = threadIdx.x; e0 < npad * kCpr; e0 += (kPjStage / 2) * kPjThreads) {
            float4 x0[kPjStage / 2], x1[kPjStage / 2];
#pragma unroll
            for (int u = 0; u < kPjStage / 2; ++u) {
                const int e = e0 + u * kPjThreads, b = e / kCpr, c = e % kCpr;
                x0[u] = x1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (b < nb) {
                    const float4* src = reinterpret_cast<const float4*>(out + ((size_t)(b0 + b) * heads + h) * ROLAQ_D_C + 8 * c);
                    x0[u] = src[0];
                    x1[u] = src[1];
                }
            }
#pragma unroll
            for (int u = 0; u < kPjStage / 2; ++u) {
                const int e = e0 + u * kPjThreads, b = e / kCpr, c = e % kCpr;
                if (b < npad)
                    *reinterpret_cast<uint4*>(&sm.b[b >> 3][c][(b & 7) * 16]) =
                        make_uint4(pack_bf16(x0[u].x, x0[u].y), pack_bf16(x0[u].z, x0[u].w),
                                   pack_bf16(x1[u].x, x1[u].y), pack_bf16(x1[u].z, x1[u].w));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (warp == 0) {
            const uint32_t idesc = proj_idesc(npad);
            const uint64_t da = smem_desc(smem_u32(sm.a[0][0]), kPjBlock, 1024, 2);
            const uint64_t db = smem_desc(smem_u32(&sm.b[0][0][0]), 128, (ROLAQ_D_C / 8) * 128, 0);
            bool ok = true;
            for (int kc = 0; kc < kChunks && ok; ++kc) {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full[kc]), 0, &sm.abort));
                if (ok) {
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int s = 0; s < 8; ++s) {
                            const int ks = 8 * kc + s;
                            umma_ss1(tmem, da + (uint64_t)((kc * 2 * kPjBlock + s * 2048) >> 4),
                                     db + (uint64_t)((ks * 256) >> 4), idesc, ks > 0 ? 1u : 0u);
                        }
                    }
                    __syncwarp();
                }
            }
            if (ok) {
                if (elect_one()) umma_commit(smem_u32(&sm.mma));
                __syncwarp();
            }
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.mma), (unsigned)(it & 1), &sm.abort));
        tc_fence_after();
        if (ok) {
            float* dst = v + (size_t)h * ROLAQ_D_V + m;
            proj_epilogue(tmem, warp, npad, [&](int b, float x) {
                if (b < nb) dst[(size_t)(b0 + b) * heads * ROLAQ_D_V] = x;
            });
        }
        tc_fence_before();
        __syncthreads();
        if (sm.abort) break;
    }
    tc_fence_after();
    if (warp == 0) proj_tmem_free(tmem);
}

}  // namespace rolaq
