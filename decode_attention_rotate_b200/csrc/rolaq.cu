// librolaq: C ABI over the sm_100a kernels of the 2-bit rotated MLA cache.
// One translation unit so the device status word is a single symbol.
#include <math.h>
#include <stdio.h>
#include <string.h>
#include <mutex>

#include "common.cuh"
#include "decode.cuh"
#include "decode_bf16.cuh"
#include "project.cuh"
#include "quantize.cuh"

using namespace rolaq;

namespace {

constexpr int kVersion = 100;   // 0.1.0
constexpr int kMaxDevices = 64;

int device_sms(int dev) {
    static int cache[kMaxDevices] = {0};
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

int current_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return device_sms(dev);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, void* base, uint64_t inner, uint64_t rows,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Launch as a programmatic dependent of the previous kernel in the stream (the kernel
// itself waits with griddepcontrol.wait before it touches memory the previous one may use).
extern "C++" {
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
}  // extern "C++"

int check_cache(const rolaq_cache* c) {
    if (!c || !c->pages_dev || !c->page_table_dev || c->num_pages <= 0 || c->batch <= 0 ||
        c->max_pages_per_seq <= 0)
        return ROLAQ_EINVAL;
    if (!aligned(c->pages_dev, 256) || !aligned(c->page_table_dev, 4)) return ROLAQ_EINVAL;
    if (c->n_sink < 0 || c->n_recent < 0) return ROLAQ_EINVAL;
    if ((c->n_sink > 0 || c->n_recent > 0) && (!c->prot_dev || !aligned(c->prot_dev, 16)))
        return ROLAQ_EINVAL;
    if (c->num_pages * (int64_t)(ROLAQ_PAGE_BYTES / 128) >= (int64_t)INT32_MAX) return ROLAQ_EINVAL;
    return ROLAQ_OK;
}

int check_params(const rolaq_layer_params* p) {
    if (!p || !(p->tau > 0.f) || !(p->gain > 0.f) || !isfinite(p->tau) || !isfinite(p->gain) ||
        !(p->level_a > 0.f) || !(p->level_b > p->level_a))
        return ROLAQ_EINVAL;
    return ROLAQ_OK;
}

// Split-K target: one work item per SM.  Every head chunk of an item is its own CTA,
// so with more heads the items run as several waves of equally sized CTAs.
int decode_target_items() { return current_sms(); }

// Scratch per work item: its partial O and (m, l) for every head.
size_t decode_item_bytes(int heads) { return (size_t)heads * (ROLAQ_D_C * sizeof(float) + sizeof(float2)); }

size_t decode_ws_bytes_for(int batch, int heads, int target) {
    return ((size_t)target + (size_t)batch) * decode_item_bytes(heads);
}

size_t decode_ws_bytes(int batch, int heads) { return decode_ws_bytes_for(batch, heads, decode_target_items()); }

// Fused append: the new tokens' rotated coordinates, fp32 [batch][512].
size_t decode_append_ws_bytes(int batch) { return (size_t)batch * ROLAQ_D_C * sizeof(float); }

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
void set_smem_limit_once(Kernel k, size_t smem, bool* done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
    if (!done[dev]) {
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        done[dev] = true;
    }
}

int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ROLAQ_OK : ROLAQ_ECUDA;
}

}  // namespace

extern "C" {

int rolaq_version(void) { return kVersion; }

const char* rolaq_strerror(int code) {
    switch (code) {
        case ROLAQ_OK: return "ok";
        case ROLAQ_EINVAL: return "invalid argument (null or misaligned pointer, bad size or shape)";
        case ROLAQ_ENOSPACE: return "workspace too small";
        case ROLAQ_ECUDA: return "CUDA call failed";
        case ROLAQ_EUNSUPPORTED: return "unsupported shape";
        default: return "unknown error";
    }
}

int rolaq_layer_params_init(rolaq_layer_params* p, float tau, float gain) {
    if (!p || !isfinite(tau) || !isfinite(gain) || !(tau > 0.f) || !(gain > 0.f)) return ROLAQ_EINVAL;
    const double t = tau;
    const double inv_sqrt_2pi = 0.39894228040143267794;
    const double phi0 = inv_sqrt_2pi, phit = inv_sqrt_2pi * exp(-0.5 * t * t);
    const double Phit = 0.5 * (1.0 + erf(t / sqrt(2.0)));
    const double a = (phi0 - phit) / (Phit - 0.5);
    const double b = phit / (0.5 * erfc(t / sqrt(2.0)));
    p->tau = tau;
    p->gain = gain;
    p->level_a = (float)a;
    p->level_b = (float)b;
    return ROLAQ_OK;
}

int rolaq_coupled_gain(float tau, double* gain, double* kappa1) {
    if (!gain || !isfinite(tau) || !(tau > 0.f)) return ROLAQ_EINVAL;
    const double t = tau;
    const double inv_sqrt_2pi = 0.39894228040143267794;
    const double phi0 = inv_sqrt_2pi, phit = inv_sqrt_2pi * exp(-0.5 * t * t);
    const double a = (phi0 - phit) / (0.5 * erf(t / sqrt(2.0)));
    const double b = phit / (0.5 * erfc(t / sqrt(2.0)));
    const double k1 = 2.0 * (a * (phi0 - phit) + b * phit);
    *gain = 1.0 / k1;
    if (kappa1) *kappa1 = k1;
    return ROLAQ_OK;
}

int rolaq_prepare_rotation(const float* R_dev, void* R_split_dev, void* stream) {
    if (!R_dev || !R_split_dev || !aligned(R_dev, 4) || !aligned(R_split_dev, 16)) return ROLAQ_EINVAL;
    rolaq_split_rotation<<<ROLAQ_D_C, 128, 0, (cudaStream_t)stream>>>(
        R_dev, reinterpret_cast<__nv_bfloat16*>(R_split_dev));
    return launch_status();
}

int rolaq_quantize_append(const rolaq_cache* cache, const rolaq_layer_params* p,
                          const void* R_split_dev, const void* c_dev, const void* k_R_dev,
                          const int32_t* req_dev, const int32_t* pos_dev,
                          const int32_t* seq_lens_dev, int n, void* stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if ((rc = check_params(p))) return rc;
    if (n < 0) return ROLAQ_EINVAL;
    if (n == 0) return ROLAQ_OK;
    if (!R_split_dev || !c_dev || !k_R_dev || !req_dev || !pos_dev) return ROLAQ_EINVAL;
    if (!aligned(R_split_dev, 16) || !aligned(c_dev, 16) || !aligned(k_R_dev, 16) ||
        !aligned(req_dev, 4) || !aligned(pos_dev, 4))
        return ROLAQ_EINVAL;
    if (cache->n_recent > 0 && !seq_lens_dev) return ROLAQ_EINVAL;

    if (n <= kSmallMaxN) {
        QuantArgs a;
        a.pages = reinterpret_cast<uint8_t*>(cache->pages_dev);
        a.num_pages = cache->num_pages;
        a.page_table = cache->page_table_dev;
        a.max_pages = cache->max_pages_per_seq;
        a.batch = cache->batch;
        a.prot = (cache->n_sink + cache->n_recent > 0) ? reinterpret_cast<__nv_bfloat16*>(cache->prot_dev) : nullptr;
        a.n_sink = cache->n_sink;
        a.n_recent = cache->n_recent;
        a.req = req_dev;
        a.pos = pos_dev;
        a.seq_lens = seq_lens_dev;
        a.k_r = reinterpret_cast<const __nv_bfloat16*>(k_R_dev);
        a.n = n;
        a.tau = p->tau;
        a.gain = p->gain;
        dim3 grid(kSmallSlices, ROLAQ_GROUPS, (n + kSmallTok - 1) / kSmallTok);
        rolaq_quantize_small_kernel<<<grid, kSmallThreads, 0, (cudaStream_t)stream>>>(
            reinterpret_cast<const __nv_bfloat16*>(R_split_dev), reinterpret_cast<const __nv_bfloat16*>(c_dev), a);
        return launch_status();
    }

    CUtensorMap map_c, map_r;
    if (!encode_2d(&map_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(c_dev), ROLAQ_D_C,
                   (uint64_t)n, ROLAQ_D_C * 2, kQK, kQTileM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&map_r, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(R_split_dev), ROLAQ_D_C,
                   kQPlanes * ROLAQ_D_C, ROLAQ_D_C * 2, kQK, kQN, CU_TENSOR_MAP_SWIZZLE_128B))
        return ROLAQ_ECUDA;

    QuantArgs a;
    a.pages = reinterpret_cast<uint8_t*>(cache->pages_dev);
    a.num_pages = cache->num_pages;
    a.page_table = cache->page_table_dev;
    a.max_pages = cache->max_pages_per_seq;
    a.batch = cache->batch;
    a.prot = (cache->n_sink + cache->n_recent > 0) ? reinterpret_cast<__nv_bfloat16*>(cache->prot_dev) : nullptr;
    a.n_sink = cache->n_sink;
    a.n_recent = cache->n_recent;
    a.req = req_dev;
    a.pos = pos_dev;
    a.seq_lens = seq_lens_dev;
    a.k_r = reinterpret_cast<const __nv_bfloat16*>(k_R_dev);
    a.n = n;
    a.tau = p->tau;
    a.gain = p->gain;

    const size_t smem = sizeof(QuantSmem) + 1024;
    static bool attr_done[kMaxDevices] = {false};
    set_smem_limit_once(rolaq_quantize_kernel, smem, attr_done);
    // one CTA per SM, or two per tile for calls of fewer tiles than half the SMs (the
    // kernel then splits every tile's groups between a pair of CTAs)
    const int tiles = (n + kQTileM - 1) / kQTileM;
    const int grid = 2 * tiles < current_sms() ? 2 * tiles : current_sms();
    if (launch_dependent(rolaq_quantize_kernel, dim3(grid), dim3(kQThreads), smem, (cudaStream_t)stream, map_c, map_r,
                         a) != cudaSuccess)
        return ROLAQ_ECUDA;
    return launch_status();
}

size_t rolaq_decode_workspace_bytes(int batch, int heads) {
    if (batch <= 0 || heads <= 0 || heads % 16) return 0;
    return decode_ws_bytes(batch, heads);
}

// Argument checks shared by both decode entry points (everything but the workspace).
static int decode_check(const rolaq_cache* cache, const rolaq_layer_params* p, const void* q_c_rot_dev,
                        const void* q_R_dev, const int32_t* seq_lens_dev, int batch, int heads,
                        float sm_scale, const float* out_dev, const float* lse_dev) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if ((rc = check_params(p))) return rc;
    if (heads <= 0 || heads % 16) return ROLAQ_EUNSUPPORTED;
    if (batch <= 0 || batch > cache->batch) return ROLAQ_EINVAL;
    if (!q_c_rot_dev || !q_R_dev || !seq_lens_dev || !out_dev) return ROLAQ_EINVAL;
    if (!aligned(q_c_rot_dev, 4) || !aligned(q_R_dev, 4) || !aligned(seq_lens_dev, 4) ||
        !aligned(out_dev, 16) || (lse_dev && !aligned(lse_dev, 4)))
        return ROLAQ_EINVAL;
    if (!isfinite(sm_scale)) return ROLAQ_EINVAL;
    return ROLAQ_OK;
}


// The new tokens of a fused append: rotation planes, latents, RoPE keys (all null: none).
struct NewTokens {
    const void* R_split;
    const void* c;
    const void* k_r;
};

// The decode with an explicit split-K target (work items before the per-request
// remainders); the workspace must hold (target + batch) items, plus batch x 512 floats
// of rotated new-token coordinates with a fused append.
static int decode_attn_impl(const rolaq_cache* cache, const rolaq_layer_params* p,
                            const void* q_c_rot_dev, const void* q_R_dev,
                            const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                            float* out_dev, float* lse_dev,
                            void* workspace_dev, size_t workspace_bytes, void* stream, int target,
                            const NewTokens& nt = NewTokens{nullptr, nullptr, nullptr}, bool bf16 = false) {
    int rc = decode_check(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev, lse_dev);
    if (rc) return rc;
    const int nslot = cache->n_sink + cache->n_recent;
    if (bf16 && (!cache->prot_dev || nslot <= 0)) return ROLAQ_EINVAL;
    if (bf16 && (cache->n_sink % ROLAQ_PAGE_TOKENS || cache->n_recent % ROLAQ_PAGE_TOKENS)) return ROLAQ_EUNSUPPORTED;
    const bool append = nt.R_split != nullptr;
    if (append && (!nt.c || !nt.k_r || !aligned(nt.R_split, 16) || !aligned(nt.c, 16) || !aligned(nt.k_r, 16)))
        return ROLAQ_EINVAL;
    if (!workspace_dev || !aligned(workspace_dev, 16)) return ROLAQ_EINVAL;
    if (target < 1) return ROLAQ_ENOSPACE;
    const size_t ws_items = decode_ws_bytes_for(batch, heads, target);
    if (workspace_bytes < ws_items + (append ? decode_append_ws_bytes(batch) : 0)) return ROLAQ_ENOSPACE;

    // The pool as rows of 128 B; one box is a whole page (144 rows).
    CUtensorMap map_page;
    const uint64_t rows = (uint64_t)cache->num_pages * (ROLAQ_PAGE_BYTES / 128);
    if (!encode_2d(&map_page, CU_TENSOR_MAP_DATA_TYPE_UINT8, cache->pages_dev, 128, rows, 128, 128,
                   ROLAQ_PAGE_BYTES / 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return ROLAQ_ECUDA;

    const int items_cap = target + batch;
    DecodeArgs a;
    a.page_table = cache->page_table_dev;
    a.num_pages = cache->num_pages;
    a.max_pages = cache->max_pages_per_seq;
    a.prot = reinterpret_cast<const __nv_bfloat16*>(cache->prot_dev);
    a.n_sink = cache->n_sink;
    a.n_recent = cache->n_recent;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q_c_rot_dev);
    a.qr = reinterpret_cast<const __nv_bfloat16*>(q_R_dev);
    a.seq_lens = seq_lens_dev;
    a.batch = batch;
    a.heads = heads;
    a.scale_log2 = sm_scale * 1.4426950408889634f;
    a.level_a = p->level_a;
    a.level_b = p->level_b;
    a.target_items = target;
    a.ws_o = reinterpret_cast<float*>(workspace_dev);
    a.ws_ml = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(workspace_dev) +
                                        (size_t)items_cap * heads * ROLAQ_D_C * sizeof(float));
    a.append = append ? 1 : 0;
    a.app_R = reinterpret_cast<const __nv_bfloat16*>(nt.R_split);
    a.app_c = reinterpret_cast<const __nv_bfloat16*>(nt.c);
    a.ws_y = append ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace_dev) + ws_items) : nullptr;
    AppendArgs ap;
    ap.y = a.ws_y;
    ap.k_r = reinterpret_cast<const __nv_bfloat16*>(nt.k_r);
    ap.q = a.q;
    ap.qr = a.qr;
    ap.scale_log2 = a.scale_log2;
    ap.tau = p->tau;
    ap.gain = p->gain;
    ap.level_a = p->level_a;
    ap.level_b = p->level_b;
    ap.pages = reinterpret_cast<uint8_t*>(cache->pages_dev);
    ap.page_table = cache->page_table_dev;
    ap.num_pages = cache->num_pages;
    ap.max_pages = cache->max_pages_per_seq;
    ap.prot = (cache->n_sink + cache->n_recent > 0) ? reinterpret_cast<__nv_bfloat16*>(cache->prot_dev) : nullptr;
    ap.n_sink = cache->n_sink;
    ap.n_recent = cache->n_recent;

    cudaStream_t s = (cudaStream_t)stream;
    if (bf16) {
        // the side store as rows of 512 bf16 (boxes of 64 x 64, 128-byte swizzle) and the
        // pool as rows of 128 B (boxes of the 64 RoPE rows of a page)
        CUtensorMap map_x, map_kr;
        if (!encode_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cache->prot_dev, ROLAQ_D_C,
                       (uint64_t)cache->batch * nslot, ROLAQ_D_C * 2, 64, ROLAQ_PAGE_TOKENS, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_2d(&map_kr, CU_TENSOR_MAP_DATA_TYPE_UINT8, cache->pages_dev, 128, rows, 128, 128,
                       ROLAQ_PAGE_TOKENS, CU_TENSOR_MAP_SWIZZLE_128B))
            return ROLAQ_ECUDA;
        if (heads % 32 == 0) {
            const size_t smem = sizeof(Bf16Smem<32>) + 1024;
            static bool attr_done[kMaxDevices] = {false};
            set_smem_limit_once(rolaq_decode_bf16<32>, smem, attr_done);
            if (launch_dependent(rolaq_decode_bf16<32>, dim3(items_cap, heads / 32), dim3(kBf16Threads), smem, s,
                                 map_x, map_kr, a) != cudaSuccess)
                return ROLAQ_ECUDA;
        } else {
            const size_t smem = sizeof(Bf16Smem<16>) + 1024;
            static bool attr_done[kMaxDevices] = {false};
            set_smem_limit_once(rolaq_decode_bf16<16>, smem, attr_done);
            if (launch_dependent(rolaq_decode_bf16<16>, dim3(items_cap, heads / 16), dim3(kBf16Threads), smem, s,
                                 map_x, map_kr, a) != cudaSuccess)
                return ROLAQ_ECUDA;
        }
    } else if (heads % 32 == 0) {
        // 32 heads per CTA (twice the work per tensor-core instruction and per
        // dequantised tile)
        const size_t smem = sizeof(DecodeSmem<32>) + 1024;
        static bool attr_done[kMaxDevices] = {false};
        set_smem_limit_once(rolaq_decode_split<32>, smem, attr_done);
        if (launch_dependent(rolaq_decode_split<32>, dim3(items_cap, heads / 32), dim3(kDecodeThreads), smem, s,
                             map_page, a) != cudaSuccess)
            return ROLAQ_ECUDA;
    } else {
        const size_t smem = sizeof(DecodeSmem<16>) + 1024;
        static bool attr_done[kMaxDevices] = {false};
        set_smem_limit_once(rolaq_decode_split<16>, smem, attr_done);
        if (launch_dependent(rolaq_decode_split<16>, dim3(items_cap, heads / 16), dim3(kDecodeThreads), smem, s,
                             map_page, a) != cudaSuccess)
            return ROLAQ_ECUDA;
    }
    if ((rc = launch_status())) return rc;
    // the merge as a programmatic dependent of the split kernel (it waits for the split's
    // completion itself), so that its launch overlaps the split's last CTAs
    if (launch_dependent(rolaq_decode_merge, dim3(batch, heads), dim3(kMergeThreads), 0, s, (const float*)a.ws_o,
                         (const float2*)a.ws_ml, seq_lens_dev, batch, heads, target, out_dev, lse_dev, ap) != cudaSuccess)
        return ROLAQ_ECUDA;
    return launch_status();
}

int rolaq_decode_attn(const rolaq_cache* cache, const rolaq_layer_params* p,
                      const void* q_c_rot_dev, const void* q_R_dev,
                      const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                      float* out_dev, float* lse_dev,
                      void* workspace_dev, size_t workspace_bytes, void* stream) {
    return decode_attn_impl(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev,
                            lse_dev, workspace_dev, workspace_bytes, stream, decode_target_items());
}

int rolaq_decode_attn_bf16(const rolaq_cache* cache, const rolaq_layer_params* p,
                           const void* q_c_rot_dev, const void* q_R_dev,
                           const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                           float* out_dev, float* lse_dev,
                           void* workspace_dev, size_t workspace_bytes, void* stream) {
    return decode_attn_impl(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev,
                            lse_dev, workspace_dev, workspace_bytes, stream, decode_target_items(),
                            NewTokens{nullptr, nullptr, nullptr}, true);
}

size_t rolaq_decode_append_workspace_bytes(int batch, int heads) {
    const size_t base = rolaq_decode_workspace_bytes(batch, heads);
    return base ? base + decode_append_ws_bytes(batch) : 0;
}

int rolaq_decode_attn_append(const rolaq_cache* cache, const rolaq_layer_params* p,
                             const void* R_split_dev, const void* c_new_dev, const void* k_R_new_dev,
                             const void* q_c_rot_dev, const void* q_R_dev,
                             const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                             float* out_dev, float* lse_dev,
                             void* workspace_dev, size_t workspace_bytes, void* stream) {
    if (!R_split_dev || !c_new_dev || !k_R_new_dev) return ROLAQ_EINVAL;
    return decode_attn_impl(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev,
                            lse_dev, workspace_dev, workspace_bytes, stream, decode_target_items(),
                            NewTokens{R_split_dev, c_new_dev, k_R_new_dev});
}

// ---- decode with library-owned scratch -------------------------------------------
// Some callers cannot allocate device memory (a pool or captured allocator owns it, or a
// host forbids allocation after start-up), so this entry point takes the split-K scratch
// from a fixed array in the library.  The array is shared by every call on a device and
// keeps the previous call's contents; the decode kernels write every partial before the
// merge reads it, so nothing has to be cleared.  Overlapping calls race on it.
static __device__ __align__(256) unsigned char g_decode_scratch[ROLAQ_STATIC_SCRATCH_BYTES];

namespace {
// Device address of g_decode_scratch, looked up once per device with that device current
// (the host-side symbol is only a stand-in and must never reach a kernel).
void* static_scratch_ptr(int dev) {
    static void* ptrs[kMaxDevices] = {nullptr};
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}
}  // namespace

int rolaq_decode_attn_static(const rolaq_cache* cache, const rolaq_layer_params* p,
                             const void* q_c_rot_dev, const void* q_R_dev,
                             const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                             float* out_dev, float* lse_dev, void* stream) {
    int rc = decode_check(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev, lse_dev);
    if (rc) return rc;
    // as many split-K items as the fixed array holds, up to one per SM
    const long long fit = (long long)(ROLAQ_STATIC_SCRATCH_BYTES / decode_item_bytes(heads)) - batch;
    const int target = (int)(fit < decode_target_items() ? fit : decode_target_items());
    if (target < 1) return ROLAQ_ENOSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ROLAQ_ECUDA;
    void* scratch = static_scratch_ptr(dev);
    if (!scratch) return ROLAQ_ECUDA;
    return decode_attn_impl(cache, p, q_c_rot_dev, q_R_dev, seq_lens_dev, batch, heads, sm_scale, out_dev,
                            lse_dev, scratch, (size_t)ROLAQ_STATIC_SCRATCH_BYTES, stream, target);
}

int rolaq_fold_weights(const float* W_UK_dev, const float* W_UV_dev, const float* R_dev,
                       int heads, void* W_q_dev, void* W_o_dev, void* stream) {
    if (!W_UK_dev || !W_UV_dev || !R_dev || !W_q_dev || !W_o_dev || heads <= 0 || heads > 65535)
        return ROLAQ_EINVAL;
    if (!aligned(W_UK_dev, 4) || !aligned(W_UV_dev, 4) || !aligned(R_dev, 4) || !aligned(W_q_dev, 16) ||
        !aligned(W_o_dev, 16))
        return ROLAQ_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    rolaq_fold_wq<<<dim3(ROLAQ_D_C / kFoldThreads, ROLAQ_D_NOPE, heads), kFoldThreads, 0, s>>>(
        W_UK_dev, R_dev, static_cast<__nv_bfloat16*>(W_q_dev));
    rolaq_fold_wo<<<dim3(ROLAQ_D_C, heads), kFoldThreads, 0, s>>>(W_UV_dev, R_dev,
                                                                   static_cast<__nv_bfloat16*>(W_o_dev));
    return launch_status();
}

int rolaq_fold_query(const void* q_nope_dev, const void* W_q_dev, int batch, int heads, void* q_c_rot_dev,
                     void* stream) {
    if (heads <= 0 || heads > 65535 || batch < 0) return ROLAQ_EINVAL;
    if (batch == 0) return ROLAQ_OK;
    if (!q_nope_dev || !W_q_dev || !q_c_rot_dev) return ROLAQ_EINVAL;
    if (!aligned(q_nope_dev, 16) || !aligned(W_q_dev, 16) || !aligned(q_c_rot_dev, 2)) return ROLAQ_EINVAL;
    CUtensorMap map;
    if (!encode_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(W_q_dev), ROLAQ_D_C,
                   (uint64_t)heads * ROLAQ_D_NOPE, ROLAQ_D_C * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return ROLAQ_ECUDA;
    const size_t smem = sizeof(FoldQSmem) + 1024;
    static bool attr_done[kMaxDevices] = {false};
    set_smem_limit_once(rolaq_fold_query_kernel, smem, attr_done);
    if (launch_dependent(rolaq_fold_query_kernel, dim3(ROLAQ_D_C / 128, heads), dim3(kPjThreads), smem,
                         (cudaStream_t)stream, map, static_cast<const __nv_bfloat16*>(q_nope_dev), batch, heads,
                         static_cast<__nv_bfloat16*>(q_c_rot_dev)) != cudaSuccess)
        return ROLAQ_ECUDA;
    return launch_status();
}

int rolaq_unfold_output(const float* out_dev, const void* W_o_dev, int batch, int heads, float* v_dev,
                        void* stream) {
    if (heads <= 0 || heads > 65535 || batch < 0) return ROLAQ_EINVAL;
    if (batch == 0) return ROLAQ_OK;
    if (!out_dev || !W_o_dev || !v_dev) return ROLAQ_EINVAL;
    if (!aligned(out_dev, 16) || !aligned(W_o_dev, 16) || !aligned(v_dev, 4)) return ROLAQ_EINVAL;
    CUtensorMap map;
    if (!encode_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(W_o_dev), ROLAQ_D_V,
                   (uint64_t)heads * ROLAQ_D_C, ROLAQ_D_V * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return ROLAQ_ECUDA;
    const size_t smem = sizeof(UnfoldSmem) + 1024;
    static bool attr_done[kMaxDevices] = {false};
    set_smem_limit_once(rolaq_unfold_output_kernel, smem, attr_done);
    if (launch_dependent(rolaq_unfold_output_kernel, dim3(heads), dim3(kPjThreads), smem, (cudaStream_t)stream, map,
                         out_dev, batch, heads, v_dev) != cudaSuccess)
        return ROLAQ_ECUDA;
    return launch_status();
}

int rolaq_get_status(int* bits, void* stream) {
    if (!bits) return ROLAQ_EINVAL;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ROLAQ_ECUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return ROLAQ_ECUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return ROLAQ_ECUDA;
    *bits = (int)v;
    return ROLAQ_OK;
}

}  // extern "C"
