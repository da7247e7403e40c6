// fp4lin.cu -- the C ABI (include/fp4lin.h): host-side argument checks and
// launches of the quantiser, KV and GEMM kernels.  One translation unit, so
// the per-device status word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "gemm_sm100_2sm.cuh"
#include "gemm_sm100_2sm_decode.cuh"
#include "kv.cuh"
#include "kv_attention.cuh"
#include "gptq.cuh"
#include "hessian.cuh"
#include "quantize.cuh"
#include "scale_search.cuh"

using namespace fp4lin;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool probed = false;
    int status = FP4LIN_OK;
    int sms = 0;
    bool gemm_attr[7] = {false, false, false, false, false, false, false};
    int pair_clusters[4] = {0, 0, 0, 0};  // resident clusters of the pair kernels (0: not yet queried)
    bool attn_attr[KA_GMAX + 1] = {};  // dynamic shared memory raised for kv_attn_tc_kernel<G>
    bool gptq_attr = false;            // dynamic shared memory raised for gptq_update_kernel
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];

// Current device's info; FP4LIN_ERR_DEVICE unless it is compute capability 10.0.
int current_device(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return FP4LIN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    DeviceInfo &d = g_dev[dev];
    if (!d.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FP4LIN_ERR_CUDA;
        d.status = (major == 10 && minor == 0) ? FP4LIN_OK : FP4LIN_ERR_DEVICE;
        d.sms = sms;
        d.probed = true;
    }
    *out = &d;
    return d.status;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline int launch_status() { return cudaGetLastError() == cudaSuccess ? FP4LIN_OK : FP4LIN_ERR_CUDA; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over packed codes [rows, K/2] bytes; box = 128 bytes x box_rows, 128-byte swizzle,
// out-of-range rows and columns read as zero.
bool make_code_map(CUtensorMap *m, const uint8_t *codes, int64_t rows, int64_t K, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a scale buffer in the tensor-core layout, seen as rows of 256 bytes (half
// a 512-byte atom each); box = 256 bytes x box_rows, no swizzle, rows past the end read as zero.
bool make_scale_map(CUtensorMap *m, const uint8_t *scales, int64_t rows, int64_t sf_cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const int64_t bytes = (rows + 127) / 128 * 128 * ((sf_cols + 3) / 4 * 4);
    cuuint64_t dims[2] = {256u, (cuuint64_t)(bytes / 256)};
    cuuint64_t strides[1] = {256u};
    cuuint32_t box[2] = {256u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(scales), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM planning
struct GemmPlan {
    bool swap;  // decode form: the MMA runs y^T = W A^T over 128-row weight tiles
    int bn;
    int splits, kps, nk, num_mt, num_nt;
    int64_t ldw;
    size_t ws_bytes;
};

// Decode form (M <= 16): tiles of 128 weight rows, K split s ways.  s minimises the k-tiles the
// busiest CTA streams, ceil(tiles*s / sms) * ceil(nk / s), plus, for s > 1, the partial sums'
// round trip through HBM and the reduction launch, both counted in the same k-tile units
// (one unit = one 128 x 256 weight tile with its scales, ~18 KB).
GemmPlan plan_decode(int64_t M, int64_t N, int64_t K, int sms)
{
    GemmPlan p{};
    p.swap = true;
    p.bn = 16;
    p.num_mt = (int)((N + 127) / 128);
    p.num_nt = 1;
    p.nk = (int)((K + 255) / 256);
    p.ldw = (N + 3) / 4 * 4;
    double best = 1e300;
    for (int s = 1; s <= std::min(p.nk, 16); ++s) {
        const int kps = (p.nk + s - 1) / s;
        const int eff = (p.nk + kps - 1) / kps;  // splits actually used
        if (eff != s)
            continue;
        const int64_t waves = ((int64_t)p.num_mt * s + sms - 1) / sms;
        double cost = (double)(waves * kps);
        if (s > 1)
            cost += 4.0 + 2.0 * s * (double)M * (double)p.ldw * 4.0 / ((double)sms * 18432.0);
        if (cost < best) {
            best = cost;
            p.splits = s;
            p.kps = kps;
        }
    }
    p.ws_bytes = p.splits > 1 ? (size_t)p.splits * (size_t)M * (size_t)p.ldw * sizeof(float) : 0;
    return p;
}

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int sms)
{
    if (M <= 16)
        return plan_decode(M, N, K, sms);
    GemmPlan p{};
    // 128 x 256 tiles for the prefill shapes (measured faster than 128 x 192 with two
    // accumulators: 250 against 332 us on the 8192 x 14336 x 4096 product)
    p.bn = (M > 128 && N > 128) ? 256 : 64;
    p.num_mt = (int)((M + 127) / 128);
    p.num_nt = (int)((N + p.bn - 1) / p.bn);
    p.nk = (int)((K + 255) / 256);
    p.splits = 1;
    p.kps = p.nk;
    p.ldw = (N + 3) / 4 * 4;
    const int64_t tiles = (int64_t)p.num_mt * p.num_nt;
    if (tiles < sms && p.nk >= 2) {
        int s = (int)std::min<int64_t>({(int64_t)p.nk, std::max<int64_t>(1, sms / tiles), 16});
        if (s > 1) {
            const int kps = (p.nk + s - 1) / s;
            s = (p.nk + kps - 1) / kps;
            if (s > 1) {
                p.splits = s;
                p.kps = kps;
            }
        }
    }
    p.ws_bytes = p.splits > 1 ? (size_t)p.splits * (size_t)M * (size_t)p.ldw * sizeof(float) : 0;
    return p;
}

// m-tiles per raster group; FP4LIN_RASTER overrides (tuning experiments).  8: on the
// 8192 x 14336 x 4096 product, groups of 2-8 m-tiles measured 242-244 us (NVFP4), 16 255 us,
// 32-64 259-262 us.
int raster_group(int num_mt)
{
    const char *e = getenv("FP4LIN_RASTER");
    const int env = e ? atoi(e) : 0;
    const int g = env > 0 ? env : 8;
    return std::max(1, std::min(g, num_mt));
}

// Launch with programmatic stream serialisation: the kernel may start before the previous one
// in the stream has finished, and must pdl_wait before touching anything that one writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The bf16 activations a fused decode GEMM quantises itself (GemmCfg FUSEQ).
struct FuseIn {
    const void *x;
    int64_t ld;
    int had;
    const float *part;  // amax partials (npart > 0: dynamic tensor scale, written to g_out)
    int npart;
    float *g_out;
};

template <class C>
int launch_gemm_cfg(DeviceInfo *dev, int attr_slot, const GemmPlan &pl, const uint8_t *a_codes,
                    const uint8_t *a_scales, const float *g_a, const uint8_t *w_codes, const uint8_t *w_scales,
                    const float *g_w, void *y, int64_t M, int64_t N, int64_t K, int64_t ldy, float *ws,
                    cudaStream_t st, const QuantOut &qo, const FuseIn *fi = nullptr, const uint8_t *a_tiled = nullptr)
{
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (!dev->gemm_attr[attr_slot]) {
            if (cudaFuncSetAttribute(fp4_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_BYTES) != cudaSuccess)
                return FP4LIN_ERR_CUDA;
            dev->gemm_attr[attr_slot] = true;
        }
    }
    CUtensorMap tmA, tmB;
    // with tiled A the map is not used; it is built over the tiled buffer so it stays valid
    if (!make_code_map(&tmA, a_tiled ? a_tiled : a_codes, a_tiled ? (M + 127) / 128 * 128 : M, K, 128))
        return FP4LIN_ERR_CUDA;
    if (fi)
        tmB = tmA;  // not used: the kernel quantises the activations itself
    else if (!make_code_map(&tmB, w_codes, N, K, C::BN))
        return FP4LIN_ERR_CUDA;
    GemmParams p{};
    p.sfa = a_scales;
    p.sfb = w_scales;
    p.g_a = g_a;
    p.g_w = g_w;
    p.y = reinterpret_cast<__nv_bfloat16 *>(y);
    p.ws = ws;
    p.M = M;
    p.N = N;
    p.K = K;
    p.ldy = ldy;
    p.ldw = pl.ldw;
    p.katoms = C::NV ? K / 64 : (K / 32 + 3) / 4;
    p.sfb_rtiles = (N + 127) / 128;
    p.num_mt = pl.num_mt;
    p.num_nt = pl.num_nt;
    p.nk = pl.nk;
    p.kps = pl.kps;
    p.splits = pl.splits;
    p.work = (int64_t)pl.num_mt * pl.num_nt * pl.splits;
    p.raster = raster_group(pl.num_mt);
    p.qc = qo.qc;
    p.qs = qo.qs;
    p.qg = qo.qg;
    p.qhad = qo.qhad;
    p.qkatoms = qo.qkatoms;
    p.a_tiled = a_tiled;
    if (fi) {
        p.xa = reinterpret_cast<const __nv_bfloat16 *>(fi->x);
        p.ld_xa = fi->ld;
        p.xhad = fi->had;
        p.xpart = fi->part;
        p.xnpart = fi->npart;
        p.g_a_out = fi->g_out;
    }
    const int grid = (int)std::min<int64_t>(p.work, dev->sms);
    if (fi && fi->npart > 0) {  // overlaps the amax pass: only the activation encoders wait for it
        if (launch_pdl(fp4_gemm_kernel<C>, grid, C::THREADS, C::SMEM_BYTES, st, tmA, tmB, p) != cudaSuccess) {
            cudaGetLastError();
            return FP4LIN_ERR_CUDA;
        }
    } else {
        fp4_gemm_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tmA, tmB, p);
    }
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    if (pl.splits > 1) {
        const int64_t rM = C::SWAP ? N : M, rN = C::SWAP ? M : N;  // the output's shape
        const int64_t items = rM * ((rN + 3) / 4);
        const int rgrid = (int)std::min<int64_t>((items + 255) / 256, (int64_t)dev->sms * 8);
        const float *ga = C::NV ? g_a : nullptr, *gw = C::NV ? g_w : nullptr;
        if (launch_pdl(splitk_reduce_kernel, rgrid, 256, 0, st, (const float *)ws, pl.splits, rM, rN, pl.ldw, ga, gw,
                       reinterpret_cast<__nv_bfloat16 *>(y), ldy, qo) != cudaSuccess) {
            cudaGetLastError();
            return FP4LIN_ERR_CUDA;
        }
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    return FP4LIN_OK;
}

// Which kernel runs a GEMM of 256-column tiles that needs no K split: the CTA-pair kernel
// (256 x 256 tiles over two SMs) once M fills a pair's 256 rows, else the one-CTA kernel;
// FP4LIN_GEMM_KERNEL=single or =pair forces one.  Both give identical results.  On the
// 8192 x 14336 x 4096 prefill product the pair takes 212 us (NVFP4) and 189 us (MXFP4)
// against the one-CTA kernel's 228 and 206 us: per SM it reads a third less operand data
// from shared memory per FLOP.
bool use_pair_kernel(const GemmPlan &pl, int64_t M)
{
    if (pl.bn != 256 || pl.splits != 1)
        return false;
    const char *e = getenv("FP4LIN_GEMM_KERNEL");
    if (e && strcmp(e, "single") == 0)
        return false;
    if (e && strcmp(e, "pair") == 0)
        return true;
    return M >= 256;
}

template <class C>
int launch_gemm_pair(DeviceInfo *dev, int slot, const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a,
                     const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w, void *y, int64_t M,
                     int64_t N, int64_t K, int64_t ldy, cudaStream_t st)
{
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (dev->pair_clusters[slot] == 0) {
            if (cudaFuncSetAttribute(fp4_gemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_BYTES) != cudaSuccess)
                return FP4LIN_ERR_CUDA;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)(dev->sms & ~1));
            cfg.blockDim = dim3(C::THREADS);
            cfg.dynamicSmemBytes = C::SMEM_BYTES;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, fp4_gemm_pair_kernel<C>, &cfg) != cudaSuccess || n < 1)
                return FP4LIN_ERR_CUDA;
            dev->pair_clusters[slot] = n;
        }
    }
    const int64_t sf_cols = C::NV ? K / 16 : K / 32;
    CUtensorMap tmA, tmB, tmSFA, tmSFB;
    if (!make_code_map(&tmA, a_codes, M, K, 128) || !make_code_map(&tmB, w_codes, N, K, 128) ||
        !make_scale_map(&tmSFA, a_scales, M, sf_cols, C::SF_BOX_ROWS) ||
        !make_scale_map(&tmSFB, w_scales, N, sf_cols, C::SF_BOX_ROWS))
        return FP4LIN_ERR_CUDA;
    Gemm2Params p{};
    p.g_a = g_a;
    p.g_w = g_w;
    p.y = reinterpret_cast<__nv_bfloat16 *>(y);
    p.M = M;
    p.N = N;
    p.K = K;
    p.ldy = ldy;
    p.katoms = (sf_cols + 3) / 4;
    p.num_mt = (int)((M + 255) / 256);
    p.num_nt = (int)((N + 255) / 256);
    p.nk = (int)((K + 255) / 256);
    p.work = (int64_t)p.num_mt * p.num_nt;
    p.raster = std::max(1, std::min(raster_group(2 * p.num_mt) / 2, p.num_mt));
    const int64_t clusters = std::min<int64_t>(p.work, dev->pair_clusters[slot]);
    fp4_gemm_pair_kernel<C><<<(unsigned)(2 * clusters), C::THREADS, C::SMEM_BYTES, st>>>(tmA, tmB, tmSFA, tmSFB, p);
    return launch_status();
}

// The decode GEMM (M <= 16) on CTA pairs: 256 weight rows per pair, K split s ways over the
// pairs, s chosen as plan_decode does but for pairs and only among splits whose partial sums
// fit the caller's workspace.
GemmPlan plan_decode_pair(int64_t M, int64_t N, int64_t K, int pairs, size_t ws_avail)
{
    GemmPlan p{};
    p.swap = true;
    p.bn = 16;
    p.num_mt = (int)((N + 255) / 256);
    p.num_nt = 1;
    p.nk = (int)((K + 255) / 256);
    p.ldw = (N + 3) / 4 * 4;
    p.splits = 1;
    p.kps = p.nk;
    double best = 1e300;
    for (int s = 1; s <= std::min(p.nk, 16); ++s) {
        const int kps = (p.nk + s - 1) / s;
        const int eff = (p.nk + kps - 1) / kps;
        if (eff != s)
            continue;
        const size_t need = (size_t)s * (size_t)M * (size_t)p.ldw * sizeof(float);
        if (s > 1 && need > ws_avail)
            continue;
        const int64_t waves = ((int64_t)p.num_mt * s + pairs - 1) / pairs;
        double cost = (double)(waves * kps);
        if (s > 1)
            cost += 4.0 + 2.0 * s * (double)M * (double)p.ldw * 4.0 / (2.0 * pairs * 18432.0);
        if (cost < best) {
            best = cost;
            p.splits = s;
            p.kps = kps;
        }
    }
    p.ws_bytes = p.splits > 1 ? (size_t)p.splits * (size_t)M * (size_t)p.ldw * sizeof(float) : 0;
    return p;
}

// Whether the decode GEMM runs on CTA pairs: only when FP4LIN_DECODE_KERNEL=pair asks for it.
// Both forms give the same results; the one-CTA form measured faster (16x14336x4096: 15.0
// against 16.5 us), although the pair issues half the tcgen05 instructions per weight row.
bool use_decode_pair()
{
    const char *e = getenv("FP4LIN_DECODE_KERNEL");
    return e && strcmp(e, "pair") == 0;
}

template <bool NV>
int launch_decode_pair(DeviceInfo *dev, const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a,
                       const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w, void *y, int64_t M,
                       int64_t N, int64_t K, int64_t ldy, void *workspace, size_t workspace_bytes, cudaStream_t st)
{
    using C = GemmDecodePairCfg<NV>;
    const int slot = NV ? 2 : 3;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (dev->pair_clusters[slot] == 0) {
            if (cudaFuncSetAttribute(fp4_gemm_decode_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_BYTES) != cudaSuccess)
                return FP4LIN_ERR_CUDA;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)(dev->sms & ~1));
            cfg.blockDim = dim3(C::THREADS);
            cfg.dynamicSmemBytes = C::SMEM_BYTES;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, fp4_gemm_decode_pair_kernel<C>, &cfg) != cudaSuccess || n < 1)
                return FP4LIN_ERR_CUDA;
            dev->pair_clusters[slot] = n;
        }
    }
    const int pairs = dev->pair_clusters[slot];
    const GemmPlan pl = plan_decode_pair(M, N, K, pairs, workspace ? workspace_bytes : 0);
    const int64_t sf_cols = NV ? K / 16 : K / 32;
    CUtensorMap tmA, tmB, tmSFA, tmSFB;
    if (!make_code_map(&tmA, w_codes, N, K, 128) || !make_code_map(&tmB, a_codes, M, K, C::CN) ||
        !make_scale_map(&tmSFA, w_scales, N, sf_cols, C::SF_BOX_ROWS) ||
        !make_scale_map(&tmSFB, a_scales, M, sf_cols, C::SF_BOX_ROWS))
        return FP4LIN_ERR_CUDA;
    GemmDecodePairParams p{};
    p.g_a = g_w;  // swapped slots: the MMA's A is the weights
    p.g_w = g_a;
    p.y = reinterpret_cast<__nv_bfloat16 *>(y);
    p.ws = reinterpret_cast<float *>(workspace);
    p.Nw = N;
    p.Mact = M;
    p.K = K;
    p.ldy = ldy;
    p.ldw = pl.ldw;
    p.katoms = (sf_cols + 3) / 4;
    p.katoms_act = p.katoms;
    p.num_mt = pl.num_mt;
    p.nk = pl.nk;
    p.kps = pl.kps;
    p.splits = pl.splits;
    p.work = (int64_t)pl.num_mt * pl.splits;
    const int64_t clusters = std::min<int64_t>(p.work, pairs);
    fp4_gemm_decode_pair_kernel<C><<<(unsigned)(2 * clusters), C::THREADS, C::SMEM_BYTES, st>>>(tmA, tmB, tmSFA, tmSFB,
                                                                                               p);
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    if (pl.splits > 1) {
        const int64_t items = M * ((N + 3) / 4);
        const int rgrid = (int)std::min<int64_t>((items + 255) / 256, (int64_t)dev->sms * 8);
        if (launch_pdl(splitk_reduce_kernel, rgrid, 256, 0, st, (const float *)workspace, pl.splits, M, N, pl.ldw,
                       NV ? g_w : nullptr, NV ? g_a : nullptr, reinterpret_cast<__nv_bfloat16 *>(y), ldy,
                       QuantOut{}) != cudaSuccess) {
            cudaGetLastError();
            return FP4LIN_ERR_CUDA;
        }
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    return FP4LIN_OK;
}

int gemm_entry(bool nv, const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a, const uint8_t *w_codes,
               const uint8_t *w_scales, const float *g_w, void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
               void *workspace, size_t workspace_bytes, void *stream, const QuantOut &qo = QuantOut{},
               bool w_tiled = false)
{
    const bool quant = qo.qc != nullptr;
    if (w_tiled && M > 16)  // the tile-order weights serve the decode (swapped) form only
        return (M < 1 || !a_codes) ? FP4LIN_ERR_INVALID_ARGUMENT : FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!a_codes || !a_scales || !w_codes || !w_scales || (!y && !quant) || (nv && (!g_a || !g_w)))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (quant && (!qo.qs || !qo.qg || (qo.qhad != 0 && qo.qhad != 16)))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (M < 1 || N < 1 || K < 1 || (y && ldy < N))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (K % 64 != 0 || (y && ldy % 8 != 0) || (quant && N % 64 != 0) || M > INT32_MAX / 2 || N > INT32_MAX / 2 ||
        K > INT32_MAX / 2)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(a_codes, 16) || !aligned(w_codes, 16) || !aligned(a_scales, 16) || !aligned(w_scales, 16) ||
        !aligned(y, 16) || (nv && (!aligned(g_a, 4) || !aligned(g_w, 4))) ||
        (workspace && !aligned(workspace, 16)) ||
        (quant && (!aligned(qo.qc, 16) || !aligned(qo.qs, 16) || !aligned(qo.qg, 4))))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    GemmPlan pl = plan_gemm(M, N, K, dev->sms);
    if (pl.splits > 1 && (!workspace || workspace_bytes < pl.ws_bytes)) {  // no room: run unsplit
        pl.splits = 1;
        pl.kps = pl.nk;
    }
    float *ws = reinterpret_cast<float *>(workspace);
    cudaStream_t s = as_stream(stream);
    if (pl.swap && !quant && !w_tiled && use_decode_pair()) {  // CTA pairs (opt-in): half the issue per weight row
        if (nv)
            return launch_decode_pair<true>(dev, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y, M, N, K, ldy,
                                            workspace, workspace_bytes, s);
        return launch_decode_pair<false>(dev, a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, y, M, N, K, ldy,
                                         workspace, workspace_bytes, s);
    }
    if (pl.swap) {  // the weights take the MMA's M side: operands and shapes swap places
        if (nv)
            return launch_gemm_cfg<GemmCfg<16, true, true>>(dev, 4, pl, w_codes, w_scales, g_w, a_codes, a_scales,
                                                            g_a, y, N, M, K, ldy, ws, s, qo, nullptr,
                                                            w_tiled ? w_codes : nullptr);
        return launch_gemm_cfg<GemmCfg<16, false, true>>(dev, 5, pl, w_codes, w_scales, nullptr, a_codes, a_scales,
                                                         nullptr, y, N, M, K, ldy, ws, s, qo);
    }
    if (!quant && use_pair_kernel(pl, M)) {
        if (nv)
            return launch_gemm_pair<Gemm2Cfg<true>>(dev, 0, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y, M, N,
                                                    K, ldy, s);
        return launch_gemm_pair<Gemm2Cfg<false>>(dev, 1, a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, y,
                                                 M, N, K, ldy, s);
    }
    if (nv) {
        if (pl.bn == 256)
            return launch_gemm_cfg<GemmCfg<256, true>>(dev, 0, pl, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y,
                                                       M, N, K, ldy, ws, s, qo);
        return launch_gemm_cfg<GemmCfg<64, true>>(dev, 1, pl, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y, M,
                                                  N, K, ldy, ws, s, qo);
    }
    if (pl.bn == 256)
        return launch_gemm_cfg<GemmCfg<256, false>>(dev, 2, pl, a_codes, a_scales, nullptr, w_codes, w_scales,
                                                     nullptr, y, M, N, K, ldy, ws, s, qo);
    return launch_gemm_cfg<GemmCfg<64, false>>(dev, 3, pl, a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, y,
                                                M, N, K, ldy, ws, s, qo);
}

// ------------------------------------------------------------------ quantiser helpers
int check_quant_args(const void *x, int64_t rows, int64_t cols, int64_t ld_x, const uint8_t *codes,
                     const uint8_t *scales)
{
    if (!x || !codes || !scales)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (rows < 1 || cols < 1 || ld_x < cols)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (cols % 64 != 0 || ld_x % 8 != 0 || (rows + QROWS - 1) / QROWS > 65535)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16))
        return FP4LIN_ERR_MISALIGNED;
    return FP4LIN_OK;
}

// quantiser grid: x = segments of 32 blocks, y = groups of QROWS rows
dim3 quant_grid(const QuantShape &q)
{
    return dim3((unsigned)((q.blocks_per_row + 31) / 32), (unsigned)((q.rows + QROWS - 1) / QROWS));
}

// amax pass: the same mapping, grid-strided down to at most AMAX_MAX_BLOCKS CTAs
dim3 amax_grid(const QuantShape &q)
{
    const dim3 full = quant_grid(q);
    const unsigned gx = std::min<unsigned>(full.x, AMAX_MAX_BLOCKS);
    const unsigned gy = std::min<unsigned>(full.y, std::max<unsigned>(1, AMAX_MAX_BLOCKS / gx));
    return dim3(gx, gy);
}

int launch_padding(const QuantShape &q, const DeviceInfo *dev, cudaStream_t s)
{
    if (q.pad_items == 0)
        return FP4LIN_OK;
    const int64_t grid = std::min<int64_t>((q.pad_items + QTHREADS - 1) / QTHREADS, (int64_t)dev->sms * 4);
    scale_padding_kernel<<<(unsigned)grid, QTHREADS, 0, s>>>(q);
    return launch_status();
}

QuantShape make_shape(const void *x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t *codes, uint8_t *scales,
                      int block)
{
    QuantShape q{};
    q.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    q.rows = rows;
    q.cols = cols;
    q.ld = ld_x;
    q.codes = codes;
    q.scales = scales;
    q.blocks_per_row = cols / block;
    // 256-bit loads need every block start 32-byte aligned: the base and the row stride
    q.wide = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (ld_x % 16 == 0);
    q.sf_cols = cols / block;
    q.katoms = (q.sf_cols + 3) / 4;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    q.pad_items = rows_pad * q.katoms * 4 - rows * q.sf_cols;
    return q;
}

template <int G>
int launch_attn_tc(DeviceInfo *dev, dim3 grid, const KvAttnShape &a, cudaStream_t s)
{
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (!dev->attn_attr[G]) {
            if (cudaFuncSetAttribute(kv_attn_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     ka_tc_smem(G)) != cudaSuccess)
                return FP4LIN_ERR_CUDA;
            dev->attn_attr[G] = true;
        }
    }
    kv_attn_tc_kernel<G><<<grid, KA_THREADS, ka_tc_smem(G), s>>>(a);
    return launch_status();
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

int fp4lin_version(void) { return 100; }

int64_t fp4lin_scale_bytes(int64_t rows, int64_t sf_cols)
{
    if (rows < 1 || sf_cols < 1)
        return 0;
    return (rows + 127) / 128 * 128 * ((sf_cols + 3) / 4 * 4);
}

size_t nvfp4_quantize_workspace_bytes(int64_t, int64_t) { return AMAX_MAX_BLOCKS * sizeof(float); }

size_t fp4lin_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 64)
        return 0;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            sms = v;
    } else {
        cudaGetLastError();
    }
    return plan_gemm(M, N, K, sms).ws_bytes;
}

int nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard, int compute_global_scale,
                   float *g, uint8_t *codes, uint8_t *scales, void *workspace, size_t workspace_bytes, void *stream)
{
    int st = check_quant_args(x, rows, cols, ld_x, codes, scales);
    if (st != FP4LIN_OK)
        return st;
    if (!g || (hadamard != 0 && hadamard != 16) || (compute_global_scale != 0 && compute_global_scale != 1))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4))
        return FP4LIN_ERR_MISALIGNED;
    if (compute_global_scale) {
        if (!workspace || workspace_bytes < AMAX_MAX_BLOCKS * sizeof(float))
            return FP4LIN_ERR_WORKSPACE;
        if (!aligned(workspace, 4))
            return FP4LIN_ERR_MISALIGNED;
    }
    DeviceInfo *dev = nullptr;
    if ((st = current_device(&dev)) != FP4LIN_OK)
        return st;
    QuantShape q = make_shape(x, rows, cols, ld_x, codes, scales, 16);
    cudaStream_t s = as_stream(stream);
    const dim3 grid(quant_grid(q));
    float *partials = reinterpret_cast<float *>(workspace);
    int n_partials = 0;
    if (compute_global_scale) {
        const dim3 agrid = amax_grid(q);
        n_partials = (int)(agrid.x * agrid.y);
        if (hadamard)
            nvfp4_amax_kernel<true><<<agrid, QTHREADS, 0, s>>>(q, partials);
        else
            nvfp4_amax_kernel<false><<<agrid, QTHREADS, 0, s>>>(q, partials);
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    // with the computed scale the encode pass starts under the amax pass (programmatic
    // dependent launch): it issues its loads of x first and waits only to read the partials
    cudaError_t e = cudaSuccess;
    if (hadamard && compute_global_scale)
        e = launch_pdl(nvfp4_quant_kernel<true, true>, grid, QTHREADS, 0, s, q, g, (const float *)partials, n_partials);
    else if (hadamard)
        nvfp4_quant_kernel<true, false><<<grid, QTHREADS, 0, s>>>(q, g, partials, 0);
    else if (compute_global_scale)
        e = launch_pdl(nvfp4_quant_kernel<false, true>, grid, QTHREADS, 0, s, q, g, (const float *)partials,
                       n_partials);
    else
        nvfp4_quant_kernel<false, false><<<grid, QTHREADS, 0, s>>>(q, g, partials, 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FP4LIN_ERR_CUDA;
    }
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    return launch_padding(q, dev, s);
}

int nvfp4_quantize_mse(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard,
                       int compute_global_scale, float *g, uint8_t *codes, uint8_t *scales, void *workspace,
                       size_t workspace_bytes, void *stream)
{
    int st = check_quant_args(x, rows, cols, ld_x, codes, scales);
    if (st != FP4LIN_OK)
        return st;
    if (!g || (hadamard != 0 && hadamard != 16) || (compute_global_scale != 0 && compute_global_scale != 1))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4))
        return FP4LIN_ERR_MISALIGNED;
    if (compute_global_scale) {
        if (!workspace || workspace_bytes < AMAX_MAX_BLOCKS * sizeof(float))
            return FP4LIN_ERR_WORKSPACE;
        if (!aligned(workspace, 4))
            return FP4LIN_ERR_MISALIGNED;
    }
    DeviceInfo *dev = nullptr;
    if ((st = current_device(&dev)) != FP4LIN_OK)
        return st;
    QuantShape q = make_shape(x, rows, cols, ld_x, codes, scales, 16);
    cudaStream_t s = as_stream(stream);
    float *partials = reinterpret_cast<float *>(workspace);
    int n_partials = 0;
    if (compute_global_scale) {
        const dim3 agrid = amax_grid(q);
        n_partials = (int)(agrid.x * agrid.y);
        if (hadamard)
            nvfp4_amax_kernel<true><<<agrid, QTHREADS, 0, s>>>(q, partials);
        else
            nvfp4_amax_kernel<false><<<agrid, QTHREADS, 0, s>>>(q, partials);
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    // one warp per block, grid-strided over the blocks
    const int64_t nblocks = rows * (cols / 16);
    const unsigned grid = (unsigned)std::min<int64_t>((nblocks + QWARPS - 1) / QWARPS, (int64_t)dev->sms * 16);
    if (hadamard && compute_global_scale)
        nvfp4_quant_mse_kernel<true, true><<<grid, QTHREADS, 0, s>>>(q, g, partials, n_partials);
    else if (hadamard)
        nvfp4_quant_mse_kernel<true, false><<<grid, QTHREADS, 0, s>>>(q, g, partials, 0);
    else if (compute_global_scale)
        nvfp4_quant_mse_kernel<false, true><<<grid, QTHREADS, 0, s>>>(q, g, partials, n_partials);
    else
        nvfp4_quant_mse_kernel<false, false><<<grid, QTHREADS, 0, s>>>(q, g, partials, 0);
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    return launch_padding(q, dev, s);
}

static int mxfp4_quantize_rule(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard,
                               uint8_t *codes, uint8_t *scales, void *stream, bool nearest)
{
    int st = check_quant_args(x, rows, cols, ld_x, codes, scales);
    if (st != FP4LIN_OK)
        return st;
    if (hadamard != 0 && hadamard != 32)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    DeviceInfo *dev = nullptr;
    if ((st = current_device(&dev)) != FP4LIN_OK)
        return st;
    QuantShape q = make_shape(x, rows, cols, ld_x, codes, scales, 32);
    cudaStream_t s = as_stream(stream);
    const dim3 grid(quant_grid(q));
    if (hadamard && nearest)
        mxfp4_quant_kernel<true, true><<<grid, QTHREADS, 0, s>>>(q);
    else if (hadamard)
        mxfp4_quant_kernel<true, false><<<grid, QTHREADS, 0, s>>>(q);
    else if (nearest)
        mxfp4_quant_kernel<false, true><<<grid, QTHREADS, 0, s>>>(q);
    else
        mxfp4_quant_kernel<false, false><<<grid, QTHREADS, 0, s>>>(q);
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    return launch_padding(q, dev, s);
}

int mxfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard, uint8_t *codes,
                   uint8_t *scales, void *stream)
{
    return mxfp4_quantize_rule(x, rows, cols, ld_x, hadamard, codes, scales, stream, false);
}

int mxfp4_quantize_nearest(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard, uint8_t *codes,
                           uint8_t *scales, void *stream)
{
    return mxfp4_quantize_rule(x, rows, cols, ld_x, hadamard, codes, scales, stream, true);
}

int nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a, const uint8_t *w_codes,
               const uint8_t *w_scales, const float *g_w, void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
               void *workspace, size_t workspace_bytes, void *stream)
{
    return gemm_entry(true, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y, M, N, K, ldy, workspace,
                      workspace_bytes, stream);
}

int nvfp4_gemm_tiled(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a, const uint8_t *w_tiled,
                     const uint8_t *w_scales, const float *g_w, void *y, int64_t M, int64_t N, int64_t K, int64_t ldy,
                     void *workspace, size_t workspace_bytes, void *stream)
{
    return gemm_entry(true, a_codes, a_scales, g_a, w_tiled, w_scales, g_w, y, M, N, K, ldy, workspace,
                      workspace_bytes, stream, QuantOut{}, true);
}

size_t kv_attention_workspace_bytes(int B, int H, int G, int64_t L, int D)
{
    if (B < 1 || H < 1 || G < 1 || L < 1 || D < 1)
        return 0;
    const int64_t S = (L + KA_CHUNK - 1) / KA_CHUNK;
    return (size_t)B * H * S * G * (D + 2) * sizeof(float);
}

int kv_nvfp4_attention(const void *q, const uint8_t *k_codes, const uint8_t *k_scales, const float *g_k,
                       const uint8_t *v_codes, const uint8_t *v_scales, const float *g_v, int64_t L, float *out,
                       int B, int H, int G, int64_t Lcap, int D, void *workspace, size_t workspace_bytes,
                       void *stream)
{
    if (!q || !k_codes || !k_scales || !g_k || !v_codes || !v_scales || !g_v || !out)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (B < 1 || H < 1 || G < 1 || L < 1 || Lcap < L || D < 1)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (D != KA_D || G > KA_GMAX || (int64_t)B * H > 65535)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(k_scales, 8) ||
        !aligned(v_scales, 8) || !aligned(g_k, 4) || !aligned(g_v, 4) || !aligned(out, 16) ||
        (workspace && !aligned(workspace, 16)))
        return FP4LIN_ERR_MISALIGNED;
    const size_t need = kv_attention_workspace_bytes(B, H, G, L, D);
    if (!workspace || workspace_bytes < need)
        return FP4LIN_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    KvAttnShape a{};
    a.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    a.kc = k_codes;
    a.ks = k_scales;
    a.vc = v_codes;
    a.vs = v_scales;
    a.gk = g_k;
    a.gv = g_v;
    a.ws = reinterpret_cast<float *>(workspace);
    a.out = out;
    a.L = L;
    a.Lcap = Lcap;
    a.H = H;
    a.S = (int)((L + KA_CHUNK - 1) / KA_CHUNK);
    const dim3 grid((unsigned)a.S, (unsigned)(B * H));
    cudaStream_t s = as_stream(stream);
    {
        switch (G) {
        case 1: st = launch_attn_tc<1>(dev, grid, a, s); break;
        case 2: st = launch_attn_tc<2>(dev, grid, a, s); break;
        case 3: st = launch_attn_tc<3>(dev, grid, a, s); break;
        case 4: st = launch_attn_tc<4>(dev, grid, a, s); break;
        case 5: st = launch_attn_tc<5>(dev, grid, a, s); break;
        case 6: st = launch_attn_tc<6>(dev, grid, a, s); break;
        case 7: st = launch_attn_tc<7>(dev, grid, a, s); break;
        default: st = launch_attn_tc<8>(dev, grid, a, s); break;
        }
        if (st != FP4LIN_OK)
            return st;
    }
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    kv_attn_merge_kernel<<<(unsigned)((int64_t)B * H * G), KA_D, 0, s>>>(a, G);
    return launch_status();
}

// Up to this many activation values, every CTA of the fused decode GEMM computes their amax
// itself rather than waiting for a separate amax pass.
#ifndef FUSED_AMAX_MAX
#define FUSED_AMAX_MAX 16384
#endif

size_t nvfp4_linear_decode_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || M > 16 || N < 1 || K < 64)
        return 0;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            sms = v;
    } else {
        cudaGetLastError();
    }
    return AMAX_MAX_BLOCKS * sizeof(float) + plan_decode(M, N, K, sms).ws_bytes;
}

static int linear_decode_entry(const void *x, int64_t M, int64_t K, int64_t ld_x, int hadamard,
                               int compute_global_scale, float *g_a, const uint8_t *w_codes, bool tiled,
                               const uint8_t *w_scales, const float *g_w, void *y, int64_t N, int64_t ldy,
                               void *workspace, size_t workspace_bytes, void *stream)
{
    if (!x || !g_a || !w_codes || !w_scales || !g_w || !y)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (M < 1 || N < 1 || K < 1 || ld_x < K || ldy < N || (hadamard != 0 && hadamard != 16) ||
        (compute_global_scale != 0 && compute_global_scale != 1))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (M > 16 || K % 64 != 0 || ld_x % 8 != 0 || ldy % 8 != 0 || N > INT32_MAX / 2 || K > INT32_MAX / 2)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(x, 16) || !aligned(w_codes, 16) || !aligned(w_scales, 16) || !aligned(y, 16) || !aligned(g_a, 4) ||
        !aligned(g_w, 4) || (workspace && !aligned(workspace, 16)))
        return FP4LIN_ERR_MISALIGNED;
    if (compute_global_scale && (!workspace || workspace_bytes < AMAX_MAX_BLOCKS * sizeof(float)))
        return FP4LIN_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    cudaStream_t s = as_stream(stream);
    GemmPlan pl = plan_decode(M, N, K, dev->sms);
    float *part = reinterpret_cast<float *>(workspace);
    float *ws = nullptr;
    const size_t ws_have = workspace_bytes > AMAX_MAX_BLOCKS * sizeof(float)
                               ? workspace_bytes - AMAX_MAX_BLOCKS * sizeof(float) : 0;
    if (pl.splits > 1 && (!workspace || ws_have < pl.ws_bytes)) {  // no room for partial sums: run unsplit
        pl.splits = 1;
        pl.kps = pl.nk;
    }
    if (pl.splits > 1)
        ws = part + AMAX_MAX_BLOCKS;
    FuseIn fi{x, ld_x, hadamard, nullptr, 0, g_a};
    if (compute_global_scale && M * K <= FUSED_AMAX_MAX) {
        fi.npart = -1;  // each CTA takes the amax itself: cheaper than a launch for so few values
    } else if (compute_global_scale) {
        QuantShape q = make_shape(x, M, K, ld_x, nullptr, nullptr, 16);
        const dim3 agrid = amax_grid(q);
        fi.part = part;
        fi.npart = (int)(agrid.x * agrid.y);
        if (hadamard)
            nvfp4_amax_kernel<true><<<agrid, QTHREADS, 0, s>>>(q, part);
        else
            nvfp4_amax_kernel<false><<<agrid, QTHREADS, 0, s>>>(q, part);
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    // swapped form: the weights are the MMA's M side; g_w's slot carries the activations' scale
    return launch_gemm_cfg<GemmCfg<16, true, true, true>>(dev, 6, pl, w_codes, w_scales, g_w, nullptr, nullptr, g_a,
                                                           y, N, M, K, ldy, ws, s, QuantOut{}, &fi,
                                                           tiled ? w_codes : nullptr);
}

int nvfp4_linear_decode(const void *x, int64_t M, int64_t K, int64_t ld_x, int hadamard, int compute_global_scale,
                        float *g_a, const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w, void *y,
                        int64_t N, int64_t ldy, void *workspace, size_t workspace_bytes, void *stream)
{
    return linear_decode_entry(x, M, K, ld_x, hadamard, compute_global_scale, g_a, w_codes, false, w_scales, g_w, y,
                               N, ldy, workspace, workspace_bytes, stream);
}

int nvfp4_linear_decode_tiled(const void *x, int64_t M, int64_t K, int64_t ld_x, int hadamard,
                              int compute_global_scale, float *g_a, const uint8_t *w_tiled, const uint8_t *w_scales,
                              const float *g_w, void *y, int64_t N, int64_t ldy, void *workspace,
                              size_t workspace_bytes, void *stream)
{
    return linear_decode_entry(x, M, K, ld_x, hadamard, compute_global_scale, g_a, w_tiled, true, w_scales, g_w, y,
                               N, ldy, workspace, workspace_bytes, stream);
}

size_t fp4lin_tiled_weight_bytes(int64_t N, int64_t K)
{
    if (N < 1 || K < 1)
        return 0;
    return (size_t)((N + 127) / 128 * 128) * (size_t)((K + 255) / 256 * 128);
}

int fp4lin_tile_weights(const uint8_t *codes, int64_t N, int64_t K, uint8_t *tiled, void *stream)
{
    if (!codes || !tiled || N < 1 || K < 1)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (K % 64 != 0 || N > INT32_MAX / 2 || K > INT32_MAX / 2)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(codes, 16) || !aligned(tiled, 16))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    const int64_t chunks = (int64_t)(fp4lin_tiled_weight_bytes(N, K) / 16);
    const unsigned grid = (unsigned)std::min<int64_t>((chunks + 255) / 256, (int64_t)dev->sms * 16);
    weight_tile_kernel<<<grid, 256, 0, as_stream(stream)>>>(codes, N, K, tiled, chunks);
    return launch_status();
}

int nvfp4_gemm_quant(const uint8_t *a_codes, const uint8_t *a_scales, const float *g_a, const uint8_t *w_codes,
                     const uint8_t *w_scales, const float *g_w, void *y, int64_t ldy, int hadamard,
                     const float *g_y, uint8_t *y_codes, uint8_t *y_scales, int64_t M, int64_t N, int64_t K,
                     void *workspace, size_t workspace_bytes, void *stream)
{
    if (!y_codes)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    QuantOut qo{};
    qo.qc = y_codes;
    qo.qs = y_scales;
    qo.qg = g_y;
    qo.qhad = hadamard;
    qo.qkatoms = N / 64;
    int st = gemm_entry(true, a_codes, a_scales, g_a, w_codes, w_scales, g_w, y, M, N, K, y ? ldy : N, workspace,
                        workspace_bytes, stream, qo);
    if (st != FP4LIN_OK)
        return st;
    DeviceInfo *dev = nullptr;
    if ((st = current_device(&dev)) != FP4LIN_OK)
        return st;
    // rows M .. the next multiple of 128 of the output's scale layout are padding: zero them
    QuantShape q = make_shape(nullptr, M, N, N, y_codes, y_scales, 16);
    return launch_padding(q, dev, as_stream(stream));
}

int mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *w_codes, const uint8_t *w_scales,
               void *y, int64_t M, int64_t N, int64_t K, int64_t ldy, void *workspace, size_t workspace_bytes,
               void *stream)
{
    return gemm_entry(false, a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, y, M, N, K, ldy, workspace,
                      workspace_bytes, stream);
}

int kv_nvfp4_store(const void *kv_new, const int32_t *pos, const float *g, uint8_t *cache_codes,
                   uint8_t *cache_scales, int B, int H, int T, int64_t Lcap, int D, void *stream)
{
    if (!kv_new || !pos || !g || !cache_codes || !cache_scales)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (B < 1 || H < 1 || T < 1 || Lcap < 1 || D < 1)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (D % 16 != 0)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(kv_new, 16) || !aligned(cache_codes, 16) || !aligned(cache_scales, 16) || !aligned(pos, 4) ||
        !aligned(g, 4))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    KvStoreShape s{};
    s.x = reinterpret_cast<const __nv_bfloat16 *>(kv_new);
    s.pos = pos;
    s.g = g;
    s.codes = cache_codes;
    s.scales = cache_scales;
    s.B = B;
    s.H = H;
    s.T = T;
    s.D = D;
    s.Lcap = Lcap;
    s.total_chunks = (int64_t)B * H * T * (D / 8);
    const int64_t grid = std::min<int64_t>((s.total_chunks + KV_THREADS - 1) / KV_THREADS, (int64_t)dev->sms * 16);
    kv_store_kernel<<<(unsigned)grid, KV_THREADS, 0, as_stream(stream)>>>(s);
    return launch_status();
}

int kv_nvfp4_load_fp8(const uint8_t *cache_codes, const uint8_t *cache_scales, const float *g, int64_t L,
                      uint8_t *out_fp8, float *out_scale, int B, int H, int64_t Lcap, int D, void *stream)
{
    if (!cache_codes || !cache_scales || !g || !out_fp8 || !out_scale)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (B < 1 || H < 1 || L < 1 || Lcap < L || D < 1)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (D % 16 != 0)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(cache_codes, 16) || !aligned(cache_scales, 16) || !aligned(out_fp8, 16) || !aligned(g, 4) ||
        !aligned(out_scale, 4))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    if ((int64_t)B * H > 65535)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    KvLoadShape s{};
    s.codes = cache_codes;
    s.scales = cache_scales;
    s.g = g;
    s.out = out_fp8;
    s.out_scale = out_scale;
    s.L = L;
    s.Lcap = Lcap;
    s.bpr = D / 16;
    const int64_t npair = (L * s.bpr + 1) / 2;
    const int64_t want = std::max<int64_t>(1, (int64_t)dev->sms * 16 / ((int64_t)B * H));
    const int64_t gx = std::min<int64_t>((npair + KV_THREADS - 1) / KV_THREADS, want);
    // wide path: whole groups of 8 blocks per slice, every base 32-byte aligned
    const bool wide = (L * s.bpr) % 8 == 0 && (Lcap * s.bpr) % 8 == 0 && aligned(cache_codes, 32) &&
                      aligned(cache_scales, 8) && aligned(out_fp8, 32);
    if (wide) {
        const int64_t ngrp = L * s.bpr / 8;
        const int64_t gxw = std::min<int64_t>((ngrp + KV_THREADS - 1) / KV_THREADS, want);
        kv_load_fp8_wide_kernel<<<dim3((unsigned)gxw, (unsigned)(B * H)), KV_THREADS, 0, as_stream(stream)>>>(s);
    } else {
        kv_load_fp8_kernel<<<dim3((unsigned)gx, (unsigned)(B * H)), KV_THREADS, 0, as_stream(stream)>>>(s);
    }
    return launch_status();
}

int fp4lin_device_status(void *stream)
{
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess)
        return FP4LIN_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
        return FP4LIN_ERR_CUDA;
    return (int)v;
}

int fp4lin_wait_selftest(uint64_t limit_ns, int arrive, uint64_t *result, void *stream)
{
    if (!result || limit_ns < 1000ull || limit_ns > 100000000ull || (arrive != 0 && arrive != 1))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (!aligned(result, 8))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    wait_selftest_kernel<<<1, 64, 0, as_stream(stream)>>>((unsigned long long)limit_ns, arrive,
                                                          reinterpret_cast<unsigned long long *>(result));
    return launch_status();
}

int fp4lin_convert_selftest(const float *in, uint8_t *e2m1, uint8_t *e4m3, int64_t n, void *stream)
{
    if (!in || !e2m1 || !e4m3 || n < 1)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (!aligned(in, 4))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    const int64_t grid = std::min<int64_t>((n + 255) / 256, (int64_t)dev->sms * 32);
    convert_selftest_kernel<<<(unsigned)grid, 256, 0, as_stream(stream)>>>(in, e2m1, e4m3, n);
    return launch_status();
}

// ==================================================================== allocation-free variant
//
// nvfp4_quantize_noalloc: for callers that cannot allocate device memory --
// plug-ins whose host framework owns the whole device memory pool and forbids
// raw cudaMalloc, or latency-critical loops where a cudaMalloc/cudaFree would
// synchronise the device.  The per-CTA maxima of the tensor-scale pass live in
// this file-scope array instead of a caller workspace: 1024 floats (4 KB),
// held by every device that loads the library until the process exits.

}  // extern "C"

static __device__ __align__(256) float g_noalloc_partials[AMAX_MAX_BLOCKS];

namespace {

std::mutex g_noalloc_mutex;
float *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_partials on device `dev` (the current device).  In
// host code the symbol is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, once per device, and cached.
int noalloc_scratch(int dev, float **out)
{
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || p == nullptr)
            return FP4LIN_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return FP4LIN_OK;
}

}  // namespace

extern "C" {

int nvfp4_quantize_noalloc(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard, float *g,
                           uint8_t *codes, uint8_t *scales, void *stream)
{
    int st = check_quant_args(x, rows, cols, ld_x, codes, scales);
    if (st != FP4LIN_OK)
        return st;
    if (!g || (hadamard != 0 && hadamard != 16))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4))
        return FP4LIN_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    if ((st = current_device(&dev)) != FP4LIN_OK)
        return st;
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess)
        return FP4LIN_ERR_CUDA;
    float *scratch = nullptr;
    if ((st = noalloc_scratch(d, &scratch)) != FP4LIN_OK)
        return st;
    QuantShape q = make_shape(x, rows, cols, ld_x, codes, scales, 16);
    const dim3 agrid = amax_grid(q);
    const int64_t n_partials = (int64_t)agrid.x * agrid.y;
    if (n_partials > AMAX_MAX_BLOCKS)  // more partial maxima than the array holds
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = as_stream(stream);
    // every partial is written by the amax pass before the quantise pass reads it,
    // so nothing in the array has to start at zero
    if (hadamard)
        nvfp4_amax_kernel<true><<<agrid, QTHREADS, 0, s>>>(q, scratch);
    else
        nvfp4_amax_kernel<false><<<agrid, QTHREADS, 0, s>>>(q, scratch);
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    const dim3 grid(quant_grid(q));
    if (hadamard)
        nvfp4_quant_kernel<true, true><<<grid, QTHREADS, 0, s>>>(q, g, scratch, (int)n_partials);
    else
        nvfp4_quant_kernel<false, true><<<grid, QTHREADS, 0, s>>>(q, g, scratch, (int)n_partials);
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    return launch_padding(q, dev, s);
}

}  // extern "C"

// ------------------------------------------------------------------ MR-GPTQ
namespace {

// The two internal streams of one GPTQ call and the events that order them; everything is
// released when the call returns (CUDA frees a stream or event once its pending work is done).
struct GptqStreams {
    cudaStream_t user = nullptr, chain = nullptr, bulk = nullptr;
    cudaEvent_t ev[64];
    int nev = 0;
    bool joined = false;

    bool record_wait(cudaStream_t from, cudaStream_t to)  // `to` waits for the work queued on `from`
    {
        if (nev == 64) {  // reuse: a recorded event may be re-recorded once the wait is queued
            for (int i = 0; i < nev; ++i)
                cudaEventDestroy(ev[i]);
            nev = 0;
        }
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            return false;
        ev[nev++] = e;
        return cudaEventRecord(e, from) == cudaSuccess && cudaStreamWaitEvent(to, e, 0) == cudaSuccess;
    }
    bool fork(cudaStream_t u)
    {
        user = u;
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&chain, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&bulk, cudaStreamNonBlocking, least) != cudaSuccess)
            return false;
        return record_wait(user, chain) && record_wait(user, bulk);
    }
    bool order(cudaStream_t first, cudaStream_t then) { return record_wait(first, then); }
    bool join()
    {
        joined = record_wait(chain, user) && record_wait(bulk, user);
        return joined;
    }
    ~GptqStreams()
    {
        if (!joined && user && chain && bulk) {  // an error path: still leave nothing dangling in the caller's stream
            record_wait(chain, user);
            record_wait(bulk, user);
        }
        for (int i = 0; i < nev; ++i)
            cudaEventDestroy(ev[i]);
        if (chain)
            cudaStreamDestroy(chain);
        if (bulk)
            cudaStreamDestroy(bulk);
        cudaGetLastError();
    }
};

// Shared by both formats: checks, rotation, the optional tensor scale, the block sweep.
int gptq_entry(bool nv, const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard, const float *u,
               int64_t ld_u, int compute_global_scale, float *g, uint8_t *codes, uint8_t *scales, void *workspace,
               size_t workspace_bytes, void *stream, bool mse = false)
{
    const int G = nv ? 16 : 32;
    if (!w || !u || !codes || !scales || (nv && !g) || !workspace)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (N < 1 || K < 1 || ld_w < K || ld_u < K || (hadamard != 0 && hadamard != G) ||
        (compute_global_scale != 0 && compute_global_scale != 1))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (K % 64 != 0 || ld_w % 8 != 0 || ld_u % 4 != 0 || N > INT32_MAX / 2 || K > INT32_MAX / 2)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(w, 16) || !aligned(u, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(workspace, 16) ||
        (nv && !aligned(g, 4)))
        return FP4LIN_ERR_MISALIGNED;
    if (workspace_bytes < gptq_workspace_bytes(N, K))
        return FP4LIN_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (!dev->gptq_attr) {
            if (cudaFuncSetAttribute(gptq_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GQ_UPD_SMEM) !=
                cudaSuccess)
                return FP4LIN_ERR_CUDA;
            dev->gptq_attr = true;
        }
    }
    // Two streams forked from (and joined back into) the caller's: the sweep chain at the
    // highest priority, the bulk trailing corrections at the lowest, so that the latency-bound
    // sweep of superblock s+1 runs while the corrections of superblock s stream into the rest
    // of W'.  The two touch disjoint columns, and E^T alternates between two buffers.
    GptqStreams gs;
    if (!gs.fork(as_stream(stream)))
        return FP4LIN_ERR_CUDA;
    cudaStream_t s = gs.chain, bs = gs.bulk;
    GptqArgs a{};
    a.wr = reinterpret_cast<float *>(workspace);
    a.np = (N + 3) / 4 * 4;
    float *et_base = a.wr + N * K;
    float *partials = et_base + 2 * GQ_SB * a.np;
    a.et = et_base;
    a.u = u;
    a.N = N;
    a.K = K;
    a.ld_u = ld_u;
    a.g = g;
    a.codes = codes;
    a.scales = scales;
    a.katoms = (K / G + 3) / 4;
    const int64_t rblocks = N * (K / G);
    const unsigned rgrid = (unsigned)std::min<int64_t>((rblocks + 255) / 256, (int64_t)dev->sms * 16);
    if (nv) {
        if (hadamard)
            gptq_rotate_kernel<16, true><<<rgrid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(w), N, K, ld_w,
                                                               a.wr);
        else
            gptq_rotate_kernel<16, false><<<rgrid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(w), N, K,
                                                                ld_w, a.wr);
    } else {
        if (hadamard)
            gptq_rotate_kernel<32, true><<<rgrid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(w), N, K, ld_w,
                                                               a.wr);
        else
            gptq_rotate_kernel<32, false><<<rgrid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16 *>(w), N, K,
                                                                ld_w, a.wr);
    }
    if (launch_status() != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    if (nv && compute_global_scale) {  // g of the rotated W, as nvfp4_quantize computes it
        QuantShape q = make_shape(w, N, K, ld_w, nullptr, nullptr, 16);
        const dim3 agrid = amax_grid(q);
        if (hadamard)
            nvfp4_amax_kernel<true><<<agrid, QTHREADS, 0, s>>>(q, partials);
        else
            nvfp4_amax_kernel<false><<<agrid, QTHREADS, 0, s>>>(q, partials);
        gptq_tensor_scale_kernel<<<1, 256, 0, s>>>(partials, (int)(agrid.x * agrid.y), g);
        if (launch_status() != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
    }
    const unsigned bgrid = (unsigned)((N + GQ_ROWS - 1) / GQ_ROWS);
    const unsigned rtiles = (unsigned)((N + GQ_TILE - 1) / GQ_TILE);
    // corrections of columns j0 .. j0+nj-1 (E^T rows jo ..) to the columns [k0, k1)
    auto update = [&](cudaStream_t st, int64_t j0, int nj, int64_t jo, int64_t k0, int64_t k1) {
        const dim3 ugrid((unsigned)((k1 - k0 + GQ_TILE - 1) / GQ_TILE), rtiles);
        gptq_update_kernel<<<ugrid, 256, GQ_UPD_SMEM, st>>>(a, j0, nj, jo, k0, k1);
        return launch_status();
    };
    bool bulk_pending = false;
    for (int64_t s0 = 0; s0 < K; s0 += GQ_SB) {
        const int64_t s1 = std::min<int64_t>(K, s0 + GQ_SB), s2 = std::min<int64_t>(K, s1 + GQ_SB);
        a.et = et_base + ((s0 / GQ_SB) & 1) * GQ_SB * a.np;
        for (int64_t c0 = s0; c0 < s1; c0 += GQ_B) {
            if (nv && mse)
                gptq_block_kernel<true, true><<<bgrid, GQ_ROWS, 0, s>>>(a, c0, s0);
            else if (nv)
                gptq_block_kernel<true><<<bgrid, GQ_ROWS, 0, s>>>(a, c0, s0);
            else
                gptq_block_kernel<false><<<bgrid, GQ_ROWS, 0, s>>>(a, c0, s0);
            if (launch_status() != FP4LIN_OK)
                return FP4LIN_ERR_CUDA;
            if (c0 + GQ_B < s1 && update(s, c0, GQ_B, c0 - s0, c0 + GQ_B, s1) != FP4LIN_OK)  // rest of the superblock
                return FP4LIN_ERR_CUDA;
        }
        if (s1 == K)
            break;
        // the next superblock's columns: after the previous superblock's bulk corrections
        if (bulk_pending && !gs.order(bs, s))
            return FP4LIN_ERR_CUDA;
        if (update(s, s0, (int)(s1 - s0), 0, s1, s2) != FP4LIN_OK)
            return FP4LIN_ERR_CUDA;
        // everything after it, on the bulk stream, once this superblock's errors are written
        if (s2 < K) {
            if (!gs.order(s, bs) || update(bs, s0, (int)(s1 - s0), 0, s2, K) != FP4LIN_OK)
                return FP4LIN_ERR_CUDA;
            bulk_pending = true;
        }
    }
    if (launch_padding(make_shape(nullptr, N, K, K, codes, scales, G), dev, s) != FP4LIN_OK)
        return FP4LIN_ERR_CUDA;
    return gs.join() ? FP4LIN_OK : FP4LIN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t gptq_workspace_bytes(int64_t N, int64_t K)
{
    if (N < 1 || K < 1)
        return 0;
    return (size_t)(N * K + 2 * GQ_SB * ((N + 3) / 4 * 4) + AMAX_MAX_BLOCKS) * sizeof(float);
}

int nvfp4_gptq_quantize(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard, const float *u,
                        int64_t ld_u, int compute_global_scale, float *g, uint8_t *codes, uint8_t *scales,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    return gptq_entry(true, w, N, K, ld_w, hadamard, u, ld_u, compute_global_scale, g, codes, scales, workspace,
                      workspace_bytes, stream);
}

int nvfp4_gptq_quantize_mse(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard, const float *u,
                            int64_t ld_u, int compute_global_scale, float *g, uint8_t *codes, uint8_t *scales,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    return gptq_entry(true, w, N, K, ld_w, hadamard, u, ld_u, compute_global_scale, g, codes, scales, workspace,
                      workspace_bytes, stream, true);
}

int mxfp4_gptq_quantize(const void *w, int64_t N, int64_t K, int64_t ld_w, int hadamard, const float *u,
                        int64_t ld_u, uint8_t *codes, uint8_t *scales, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    return gptq_entry(false, w, N, K, ld_w, hadamard, u, ld_u, 0, nullptr, codes, scales, workspace,
                      workspace_bytes, stream);
}

// Workspace of gptq_hessian_factor: the rotated, column-reversed activations [T, K], the
// reversed Hessian and its factor [K, K], the factor's inverse [K, K], the inverses of its
// 64 x 64 diagonal blocks [K / 64][64][64] and one 64 x K block row of products (all binary64).
size_t gptq_hessian_workspace_bytes(int64_t T, int64_t K)
{
    if (T < 1 || K < 1 || K % HB != 0)
        return 0;
    return (size_t)(T * K + 2 * K * K + 2 * (int64_t)HB * K) * sizeof(double);
}

int gptq_hessian_factor(const double *x, int64_t T, int64_t K, int64_t ld_x, int hadamard, double damp, float *u,
                        int64_t ld_u, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!x || !u || !workspace)
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (T < 1 || K < 1 || ld_x < K || ld_u < K || (hadamard != 0 && hadamard != 16 && hadamard != 32) ||
        !(damp >= 0.0) || !(damp < 1e300))
        return FP4LIN_ERR_INVALID_ARGUMENT;
    if (K % HB != 0 || K > (int64_t)1 << 20 || T > ((int64_t)1 << 40) / K)
        return FP4LIN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(x, 8) || !aligned(u, 4) || !aligned(workspace, 16))
        return FP4LIN_ERR_MISALIGNED;
    if (workspace_bytes < gptq_hessian_workspace_bytes(T, K))
        return FP4LIN_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    int st = current_device(&dev);
    if (st != FP4LIN_OK)
        return st;
    cudaStream_t s = as_stream(stream);
    double *xr = reinterpret_cast<double *>(workspace);
    double *A = xr + T * K;                // P H P, then its Cholesky factor Lr (lower triangle)
    double *X = A + K * K;                 // Lr^-1
    double *dinv = X + K * K;              // inverses of Lr's diagonal blocks
    double *Tb = dinv + (int64_t)HB * K;   // one 64 x K block row of products
    const int nblk = (int)(K / HB);
    auto grid_for = [&](int64_t items) {
        return (unsigned)std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, (int64_t)dev->sms * 8));
    };
    // 1. rotation, columns reversed
    if (hadamard == 16)
        hess_rotate_kernel<16><<<grid_for(T * (K / 16)), 256, 0, s>>>(x, T, K, ld_x, xr);
    else if (hadamard == 32)
        hess_rotate_kernel<32><<<grid_for(T * (K / 32)), 256, 0, s>>>(x, T, K, ld_x, xr);
    else
        hess_rotate_kernel<1><<<grid_for(T * K), 256, 0, s>>>(x, T, K, ld_x, xr);
    // 2. the Gram product's lower triangle: A(m, n) = sum_t xr[t][m] xr[t][n]
    {
        DgemmArgs g{xr, xr, A, K, K, T, 1, K, 1, K, K, 0, 0, 0, 1.0, 0.0};
        dgemm_kernel<false, false, true><<<dim3(nblk, nblk, 1), 256, 0, s>>>(g);
    }
    // 3. damping
    hess_damp_kernel<<<1, 256, 0, s>>>(A, K, damp);
    // 4. blocked Cholesky, right-looking
    for (int kb = 0; kb < nblk; ++kb) {
        chol_diag_kernel<<<1, 256, 0, s>>>(A, K, kb, dinv);
        const int rem = nblk - kb - 1;
        if (rem == 0)
            break;
        chol_panel_kernel<<<rem, 256, 0, s>>>(A, K, kb, dinv);
        double *pan = A + (int64_t)(kb + 1) * HB * K + (int64_t)kb * HB;
        double *trail = A + (int64_t)(kb + 1) * HB * K + (int64_t)(kb + 1) * HB;
        DgemmArgs g{pan, pan, trail, (int64_t)rem * HB, (int64_t)rem * HB, HB, K, 1, K, 1, K, 0, 0, 0, -1.0, 1.0};
        dgemm_kernel<true, true, true><<<dim3(rem, rem, 1), 256, 0, s>>>(g);
    }
    // 5. X = Lr^-1, one block row at a time: X[i, :i] = -D_i^-1 (Lr[i, :i] X[:i, :i])
    hess_inv_init_kernel<<<grid_for(K * K), 256, 0, s>>>(X, K, dinv);
    for (int i = 1; i < nblk; ++i) {
        const int64_t w = (int64_t)i * HB;
        DgemmArgs g1{A + w * K, X, Tb, HB, w, w, K, 1, 1, K, K, 0, 0, 0, 1.0, 0.0};
        dgemm_kernel<true, false, false><<<dim3(i, 1, 1), 256, 0, s>>>(g1);
        DgemmArgs g2{dinv + (int64_t)i * HB * HB, Tb, X + w * K, HB, w, HB, HB, 1, 1, K, K, 0, 0, 0, -1.0, 0.0};
        dgemm_kernel<true, false, false><<<dim3(i, 1, 1), 256, 0, s>>>(g2);
    }
    // 6. U = P X P, upper triangle
    hess_out_kernel<<<grid_for(K * K), 256, 0, s>>>(X, K, u, ld_u);
    return cudaGetLastError() == cudaSuccess ? FP4LIN_OK : FP4LIN_ERR_CUDA;
}

}  // extern "C"
