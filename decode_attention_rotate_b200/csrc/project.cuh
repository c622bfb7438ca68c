// Absorbed projections around the cache ("RoLaQ", §3.3; Fig. 3a): the read-side rotation
// folds into the query projection and its inverse into the value projection.
//   W_q[h] = W_UK[h]^T . R     [128][512]   (once per layer)
//   W_o[h] = R^T . W_UV[h]     [512][128]   (once per layer)
//   q_c_rot[b,h] = q_nope[b,h] . W_q[h]     (per decode step, bf16 out)
//   v[b,h]       = out_rot[b,h] . W_o[h]    (per decode step, fp32 out)
// The folded weights are stored in bf16 (the precision the model's own projections carry)
// and every sum runs in fp32.  The per-step products are small and bound by reading the
// weights once: a decode step has a handful of queries per head, so each CTA splits the
// contraction over its warps (many independent 4- or 8-byte loads in flight per lane),
// keeps the weights in registers across the batch and reduces the warps' partial sums
// through shared memory in a fixed order.
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

// ---- per step: query fold ---------------------------------------------------------
// CTA = (64 output columns, head); 8 warps, warp w sums rows n = 16w .. 16w + 15 of W_q,
// lane l owns columns 2l, 2l + 1 of the CTA's 64 (one 4-byte load per row).

constexpr int kFqThreads = 256;
constexpr int kFqWarps = kFqThreads / 32;
constexpr int kFqCols = 64;
constexpr int kFqRows = ROLAQ_D_NOPE / kFqWarps;    // 16
constexpr int kFqBatch = 8;                         // queries per pass

__global__ void __launch_bounds__(kFqThreads)
rolaq_fold_query_kernel(const __nv_bfloat16* __restrict__ q_nope, const __nv_bfloat16* __restrict__ W_q,
                        int batch, int heads, __nv_bfloat16* __restrict__ q_c_rot) {
    __shared__ float s_q[kFqBatch][ROLAQ_D_NOPE];
    __shared__ float2 s_part[kFqWarps][kFqBatch][kFqCols / 2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const int col0 = blockIdx.x * kFqCols;
    const int n0 = warp * kFqRows;
    float2 w[kFqRows];
    const __nv_bfloat162* wq = reinterpret_cast<const __nv_bfloat162*>(
        W_q + ((size_t)h * ROLAQ_D_NOPE + n0) * ROLAQ_D_C + col0) + lane;
#pragma unroll
    for (int i = 0; i < kFqRows; ++i) w[i] = __bfloat1622float2(wq[(size_t)i * (ROLAQ_D_C / 2)]);
    for (int b0 = 0; b0 < batch; b0 += kFqBatch) {
        const int nb = min(kFqBatch, batch - b0);
        for (int e = threadIdx.x; e < kFqBatch * ROLAQ_D_NOPE; e += kFqThreads) {
            const int bb = e / ROLAQ_D_NOPE, n = e % ROLAQ_D_NOPE;
            s_q[bb][n] = bb < nb ? __bfloat162float(q_nope[((size_t)(b0 + bb) * heads + h) * ROLAQ_D_NOPE + n]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int bb = 0; bb < kFqBatch; ++bb) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < kFqRows; ++i) {
                const float q = s_q[bb][n0 + i];
                acc.x = fmaf(q, w[i].x, acc.x);
                acc.y = fmaf(q, w[i].y, acc.y);
            }
            s_part[warp][bb][lane] = acc;
        }
        __syncthreads();
        // 8 queries x 64 columns = 512 sums of 8 partials, two per thread
        for (int e = threadIdx.x; e < kFqBatch * kFqCols; e += kFqThreads) {
            const int bb = e / kFqCols, c = e % kFqCols;
            if (bb < nb) {
                float s = 0.f;
#pragma unroll
                for (int p = 0; p < kFqWarps; ++p) {
                    const float2 v = s_part[p][bb][c >> 1];
                    s += (c & 1) ? v.y : v.x;
                }
                q_c_rot[((size_t)(b0 + bb) * heads + h) * ROLAQ_D_C + col0 + c] = __float2bfloat16_rn(s);
            }
        }
        __syncthreads();
    }
}

// ---- per step: output unfold ------------------------------------------------------
// A cluster of 4 CTAs per head splits K = 512 into quarters.  In each CTA, warp w sums
// rows 16w .. 16w + 15 of its quarter, lane l owns columns 4l .. 4l + 3 (one 8-byte load
// per row).  The CTA reduces its warps in shared memory and stores the quarter's sums into
// the first CTA of the cluster (distributed shared memory), which adds the four quarters
// in rank order and writes v.

constexpr int kUoSplit = 4;                         // CTAs per head (cluster size)
constexpr int kUoThreads = 256;
constexpr int kUoWarps = kUoThreads / 32;
constexpr int kUoK = ROLAQ_D_C / kUoSplit;          // 128 rows of W_o per CTA
constexpr int kUoRows = kUoK / kUoWarps;            // 16 rows per warp
constexpr int kUoBatch = 4;                         // outputs per pass

__global__ void __cluster_dims__(kUoSplit, 1, 1) __launch_bounds__(kUoThreads)
rolaq_unfold_output_kernel(const float* __restrict__ out, const __nv_bfloat16* __restrict__ W_o, int batch,
                           int heads, float* __restrict__ v) {
    __shared__ float s_o[kUoBatch][kUoK];
    __shared__ float4 s_part[kUoWarps][kUoBatch][ROLAQ_D_V / 4];
    __shared__ float s_red[kUoSplit][kUoBatch][ROLAQ_D_V];   // used in the first CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const uint32_t rank = cluster_ctarank();
    const int kq = (int)rank * kUoK;                 // this CTA's quarter of K
    const int k0 = warp * kUoRows;                   // this warp's rows inside the quarter
    uint2 w[kUoRows];                                // packed bf16, widened at use
    const uint2* wo = reinterpret_cast<const uint2*>(W_o + ((size_t)h * ROLAQ_D_C + kq + k0) * ROLAQ_D_V) + lane;
#pragma unroll
    for (int i = 0; i < kUoRows; ++i) w[i] = wo[(size_t)i * (ROLAQ_D_V / 4)];
    const uint32_t red0 = mapa_shared(smem_u32(&s_red[rank][0][0]), 0);
    cluster_sync();                                  // every CTA of the cluster is running
    for (int b0 = 0; b0 < batch; b0 += kUoBatch) {
        const int nb = min(kUoBatch, batch - b0);
        for (int e = threadIdx.x; e < kUoBatch * kUoK; e += kUoThreads) {
            const int bb = e / kUoK, k = e % kUoK;
            s_o[bb][k] = bb < nb ? out[((size_t)(b0 + bb) * heads + h) * ROLAQ_D_C + kq + k] : 0.f;
        }
        __syncthreads();
        float4 acc[kUoBatch];
#pragma unroll
        for (int bb = 0; bb < kUoBatch; ++bb) acc[bb] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kUoRows; ++i) {          // widen one row, use it for every output
            const float w0 = bf16_lo(w[i].x), w1 = bf16_hi(w[i].x), w2 = bf16_lo(w[i].y), w3 = bf16_hi(w[i].y);
#pragma unroll
            for (int bb = 0; bb < kUoBatch; ++bb) {
                const float o = s_o[bb][k0 + i];
                acc[bb].x = fmaf(o, w0, acc[bb].x);
                acc[bb].y = fmaf(o, w1, acc[bb].y);
                acc[bb].z = fmaf(o, w2, acc[bb].z);
                acc[bb].w = fmaf(o, w3, acc[bb].w);
            }
        }
#pragma unroll
        for (int bb = 0; bb < kUoBatch; ++bb) s_part[warp][bb][lane] = acc[bb];
        __syncthreads();
        // the quarter's 4 x 128 sums (8 warp partials each), two per thread, into the first CTA
        for (int e = threadIdx.x; e < kUoBatch * ROLAQ_D_V; e += kUoThreads) {
            const int bb = e / ROLAQ_D_V, c = e % ROLAQ_D_V;
            float s = 0.f;
#pragma unroll
            for (int p = 0; p < kUoWarps; ++p) {
                const float4 u = s_part[p][bb][c >> 2];
                s += (c & 3) == 0 ? u.x : (c & 3) == 1 ? u.y : (c & 3) == 2 ? u.z : u.w;
            }
            st_cluster_f32(red0 + (uint32_t)e * 4u, s);
        }
        cluster_sync();                              // all quarters have landed
        if (rank == 0) {
            for (int e = threadIdx.x; e < kUoBatch * ROLAQ_D_V; e += kUoThreads) {
                const int bb = e / ROLAQ_D_V, c = e % ROLAQ_D_V;
                if (bb < nb) {
                    float s = s_red[0][bb][c];
#pragma unroll
                    for (int r = 1; r < kUoSplit; ++r) s += s_red[r][bb][c];
                    v[((size_t)(b0 + bb) * heads + h) * ROLAQ_D_V + c] = s;
                }
            }
        }
        cluster_sync();                              // the first CTA has read them (next pass reuses)
    }
}

}  // namespace rolaq
