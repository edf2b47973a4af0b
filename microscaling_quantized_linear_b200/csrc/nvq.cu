// nvq.cu -- C ABI of the microscaling-quantized linear layer (see include/nvq.h).
//
// Host side only: argument checks (nothing is launched when one fails),
// per-device capability and SM-count cache, TMA descriptor encoding through
// the driver entry point (no link-time dependency on libcuda), kernel
// launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "nvq.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "quantize.cuh"

namespace nvq {

// One status word per device (NVQ_STATUS_* bits), set by kernels, read and
// cleared by nvq_device_status().
__device__ unsigned int g_status;

// Scratch of nvfp4_quantize_noalloc: the amax pass's partial maxima.  A
// static device array, so the entry point never allocates; its device
// address is looked up by the entry point's first call on each device.
// Shared by every call on a device; fully rewritten by each call's amax pass
// before it is read.
static __device__ __align__(256) uint32_t g_noalloc_partials[NVQ_NOALLOC_MAX_PARTIALS];
// The amax pass never launches more CTAs than it has partial slots for, so
// it fits the static array too.
static_assert(kMaxAmaxPartials <= NVQ_NOALLOC_MAX_PARTIALS, "amax partials must fit the no-alloc scratch");
static_assert(kStatusTimeout == NVQ_STATUS_TIMEOUT && kStatusNonfinite == NVQ_STATUS_NONFINITE &&
                  kStatusWorkspace == NVQ_STATUS_WORKSPACE && kStatusBounds == NVQ_STATUS_BOUNDS,
              "status bits");

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool arch_ok = false;
    int num_sms = 0;
    unsigned int* status = nullptr;
    bool gemm_attr[3][3][2] = {};    // [format][BN 128/192/256][epilogue]
    bool pair_attr[3][2][2] = {};    // [format][BN 192/256][epilogue]
    bool splitk_attr[3][3][2] = {};  // [format][BN 128/192/256][receive rows 16/32]
    bool short_attr[3] = {};         // fused short-M NVFP4 kernel: [BN 128/192/256]
    // most clusters of k_split CTAs that fit on the device at once, + 1
    // (0 = not yet asked): [format][BN 128/192/256][k_split]
    int splitk_clusters[3][3][9] = {};
    bool fused_attr = false;
    int fused_occupancy = -1;        // CTAs of the one-pass quantizer per SM at its largest tile (-1: not asked)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVQ_ERR_CUDA;
        d.arch_ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        if (d.arch_ok) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return NVQ_ERR_CUDA;
            d.status = static_cast<unsigned int*>(p);
        }
        d.ready = true;
    }
    if (!d.arch_ok) return NVQ_ERR_ARCH;
    *out = &d;
    return NVQ_OK;
}

int get_encoder() {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_encode) return NVQ_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return NVQ_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return NVQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_of(int format) { return format == NVQ_NVFP4 ? 16 : 32; }
int k_multiple(int format) { return format == NVQ_NVFP4 ? 64 : 128; }

bool is_mxfp8(int format) { return format == NVQ_MXFP8 || format == NVQ_MXFP8_E5M2; }

// Checks shared by the quantizers: BF16 [rows, K] input with pitch ld.
int check_quant_shape(int format, int64_t rows, int64_t K, int64_t ld) {
    if (rows < 0 || K <= 0 || K % k_multiple(format) != 0) return NVQ_ERR_SHAPE;
    if (ld < K || ld % 8 != 0) return NVQ_ERR_SHAPE;
    if (rows * K >= (int64_t(1) << 31) || rows * ld >= (int64_t(1) << 40) || ld >= (int64_t(1) << 31))
        return NVQ_ERR_SHAPE;
    return NVQ_OK;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? NVQ_OK : NVQ_ERR_CUDA; }

// Launch with programmatic stream serialization: the grid may launch while
// the previous grid in the stream is still running.  Every kernel launched
// this way executes griddepcontrol.wait before it reads anything the
// previous grid may write, so only launch latency overlaps.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

// The amax pass: one CTA per 8 x 256 16-byte vectors, at most 8 per SM and
// at most `capacity` CTAs (one partial maximum each).
int launch_amax(const void* x, int64_t rows, int64_t K, int64_t ld, uint32_t* partial, uint32_t capacity,
                int num_sms, unsigned int* status, cudaStream_t stream, uint32_t* npartial_out) {
    const uint32_t vecs_per_row = (uint32_t)(K / 8), pitch_vecs = (uint32_t)(ld / 8);
    const uint64_t total = (uint64_t)rows * vecs_per_row;
    uint64_t want = (total + 8 * kAmaxThreads - 1) / (8 * kAmaxThreads);
    uint32_t grid = (uint32_t)(want < 1 ? 1 : want);
    uint32_t cap = (uint32_t)num_sms * 8 < (uint32_t)kMaxAmaxPartials ? (uint32_t)num_sms * 8 : kMaxAmaxPartials;
    if (cap > capacity) cap = capacity;
    if (cap == 0) return NVQ_ERR_SHAPE;
    if (grid > cap) grid = cap;
    *npartial_out = grid;
    return launch_pdl(amax_partials_kernel, dim3(grid), dim3(kAmaxThreads), 0, stream, static_cast<const uint4*>(x),
                      (uint32_t)rows, vecs_per_row, pitch_vecs, partial, capacity, status);
}

uint32_t quant_grid(uint64_t units, int num_sms) {
    uint64_t blocks = (units + kQuantThreads - 1) / kQuantThreads;
    const uint64_t cap = (uint64_t)num_sms * 6;      // 6 resident 256-thread CTAs per SM
    if (blocks > cap) blocks = cap;
    return (uint32_t)(blocks < 1 ? 1 : blocks);
}

// Limit of the kernels' pipeline waits set by nvq_set_wait_limit (0: the
// defaults, 4 s in the GEMMs and 2 s in the one-pass quantizer's barrier).
// NVQ_WAIT_LIMIT_NS in the environment sets its initial value (decimal
// nanoseconds, at most the 4 s default; anything else is ignored).
uint64_t wait_limit_from_env() {
    const char* e = getenv("NVQ_WAIT_LIMIT_NS");
    if (!e || !*e) return 0;
    char* end = nullptr;
    const unsigned long long v = strtoull(e, &end, 10);
    if (*end != '\0' || v > kWaitLimitNs) return 0;
    return (uint64_t)v;
}
std::atomic<uint64_t> g_wait_limit_ns{wait_limit_from_env()};

uint64_t pipeline_wait_ns(uint64_t dflt) {
    const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
    return v ? v : dflt;
}

constexpr size_t kFusedSmemMax = 220 * 1024;

// One-pass quantizer: opt in to its shared memory and ask how many of its
// CTAs an SM holds with the largest tile it is given (cached per device).
// Its grid barrier needs every CTA resident at once; the grid is at most one
// CTA per SM, so it runs only where that answer is at least one.
int fused_quantizer_fits(DeviceInfo* d, bool* fits) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d->fused_attr) {
        if (cudaFuncSetAttribute(nvfp4_quantize_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kFusedSmemMax + 128) != cudaSuccess) {
            cudaGetLastError();
            return NVQ_ERR_CUDA;
        }
        d->fused_attr = true;
    }
    if (d->fused_occupancy < 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_quantize_fused_kernel, kFusedThreads,
                                                          kFusedSmemMax) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        d->fused_occupancy = n;
    }
    *fits = d->fused_occupancy >= 1;
    return NVQ_OK;
}

// Dynamic NVFP4 quantization: one pass (every CTA's rows held in shared
// memory, one read of x) for tensors that fit on chip, else two passes
// (amax, then quantize with programmatic dependent launch).
// NVQ_QUANT_ONE_PASS=0 selects the two passes for every tensor.
const bool g_quant_one_pass = [] {
    const char* e = getenv("NVQ_QUANT_ONE_PASS");
    return !(e && e[0] == '0');
}();

// NVQ_GEMM_PAIRS=0 in the environment selects the one-CTA GEMM for every
// shape (the test suite runs both kernels on the same shapes).
const bool g_use_pairs = [] {
    const char* e = getenv("NVQ_GEMM_PAIRS");
    return !(e && e[0] == '0');
}();

// NVQ_GEMM_SPLITK=0 never splits K across a cluster for short M.  Split-K
// sums FP32 partials in another order, so results may differ from the
// unsplit kernel in the last bits (both within the GEMM tolerance; exact
// sums agree bit for bit).
const bool g_use_splitk = [] {
    const char* e = getenv("NVQ_GEMM_SPLITK");
    return !(e && e[0] == '0');
}();

int nvfp4_quantize_impl(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                        float* global_scale, const float* calib_amax, void* workspace, cudaStream_t stream) {
    int rc = check_quant_shape(NVQ_NVFP4, M, K, ldx);
    if (rc) return rc;
    if (M == 0) return NVQ_OK;                       // empty batch: nothing to read or write
    if (!x || !codes || !scales || !global_scale || (!workspace && !calib_amax)) return NVQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (workspace && !aligned16(workspace)))
        return NVQ_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(global_scale) & 3u) return NVQ_ERR_ALIGN;
    if (calib_amax && (reinterpret_cast<uintptr_t>(calib_amax) & 3u)) return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d))) return rc;
    const uint32_t nblk = (uint32_t)(K / 16);
    if (!calib_amax && (uint64_t)M * nblk <= kClusterMaxBlocks) {
        // small tensor: one launch of one cluster, the maximum exchanged in
        // distributed shared memory (the workspace is not touched)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kClusterCtas);
        cfg.blockDim = dim3(kClusterThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, nvfp4_quantize_cluster_kernel, static_cast<const uint16_t*>(x), (uint32_t)M, nblk,
                               (uint32_t)ldx, codes, scales, global_scale, d->status) != cudaSuccess) {
            cudaGetLastError();
            return NVQ_ERR_CUDA;
        }
        return NVQ_OK;
    }
    if (!calib_amax && g_quant_one_pass) {
        // One pass when every CTA's rows fit in shared memory (one CTA per SM,
        // at most as many CTAs as SMs).
        const int64_t rows_per_cta = (M + d->num_sms - 1) / d->num_sms;
        const size_t smem = fused_smem_bytes((size_t)rows_per_cta, (size_t)K);
        bool fits = false;
        if (smem <= kFusedSmemMax && (M + rows_per_cta - 1) / rows_per_cta <= kMaxFusedCtas &&
            rows_per_cta * (K / 16) <= (int64_t)kFusedMaxBlocks * kFusedThreads &&
            (rc = fused_quantizer_fits(d, &fits)) == NVQ_OK && fits) {
            const uint32_t grid = (uint32_t)((M + rows_per_cta - 1) / rows_per_cta);
            const uint16_t* xp = static_cast<const uint16_t*>(x);
            uint32_t rows32 = (uint32_t)M, k32 = (uint32_t)K, ld32 = (uint32_t)ldx, rpc = (uint32_t)rows_per_cta;
            unsigned long long* slots = reinterpret_cast<unsigned long long*>(
                static_cast<uint8_t*>(workspace) + kWorkspaceSlotsOffset);
            unsigned long long* gen = reinterpret_cast<unsigned long long*>(
                static_cast<uint8_t*>(workspace) + kWorkspaceGenOffset);
            uint64_t wait_ns = pipeline_wait_ns(kFusedWaitNs);
            unsigned int* status = d->status;
            void* args[] = {&xp,     &rows32, &k32, &ld32,    &rpc,   &codes, &scales,
                            &global_scale, &slots, &gen, &wait_ns, &status};
            // The kernel waits on every CTA's maximum, so every CTA must be
            // resident at once: the grid is at most one CTA per SM and an SM
            // holds one (checked above), so all of them are resident once the
            // previous grid in the stream has left the SMs.  A cooperative
            // launch would guarantee it too but costs about 2.6 us more per
            // call on B200.  Work on other streams that holds SMs past the
            // wait's limit makes the waiting CTAs read the amax from x
            // themselves: exact results, NVQ_STATUS_TIMEOUT set.
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid);
            cfg.blockDim = dim3(kFusedThreads);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelExC(&cfg, (const void*)nvfp4_quantize_fused_kernel, args) != cudaSuccess) {
                cudaGetLastError();
                return NVQ_ERR_CUDA;
            }
            return NVQ_OK;
        }
        if (rc) return rc;
    }
    uint32_t npartial = 0;
    uint32_t* partial = calib_amax ? nullptr
                                   : reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + kWorkspacePartialsOffset);
    if (!calib_amax) {
        if ((rc = launch_amax(x, M, K, ldx, partial, kMaxAmaxPartials, d->num_sms, d->status, stream, &npartial))) return rc;
    }
    const uint64_t units = (uint64_t)M * nblk;
    return launch_pdl(nvfp4_quantize_kernel, dim3(quant_grid(units, d->num_sms)), dim3(kQuantThreads), 0, stream,
                      static_cast<const uint16_t*>(x), (uint32_t)M, nblk, (uint32_t)ldx, codes, scales, global_scale,
                      partial, npartial, calib_amax, d->status);
}

int mxfp8_quantize_impl(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                        int elem, int rule, cudaStream_t stream) {
    if (!is_mxfp8(elem) || (rule != NVQ_SCALE_FLOOR && rule != NVQ_SCALE_CEIL)) return NVQ_ERR_FORMAT;
    int rc = check_quant_shape(NVQ_MXFP8, M, K, ldx);
    if (rc) return rc;
    if (M == 0) return NVQ_OK;
    if (!x || !codes || !scales) return NVQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d))) return rc;
    const uint32_t nblk = (uint32_t)(K / 32);
    const uint32_t grid = quant_grid((uint64_t)M * nblk, d->num_sms);
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    const bool e5 = elem == NVQ_MXFP8_E5M2, ceil_rule = rule == NVQ_SCALE_CEIL;
    auto kern = e5 ? (ceil_rule ? mxfp8_quantize_kernel<1, 1> : mxfp8_quantize_kernel<1, 0>)
                   : (ceil_rule ? mxfp8_quantize_kernel<0, 1> : mxfp8_quantize_kernel<0, 0>);
    return launch_pdl(kern, dim3(grid), dim3(kQuantThreads), 0, stream, xp, (uint32_t)M, nblk, (uint32_t)ldx, codes,
                      scales, d->status);
}

int encode_codes_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t kbytes, uint32_t box_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kbytes};
    const cuuint32_t box[2] = {128u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVQ_OK : NVQ_ERR_CUDA;
}

int encode_out_map(CUtensorMap* map, const void* out, int64_t rows, int64_t cols, int64_t ldo) {
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ldo * 2};
    const cuuint32_t box[2] = {32u, 32u};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(out), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVQ_OK : NVQ_ERR_CUDA;
}

// Scale buffer viewed as rows of 256 bytes; a box of box_rows rows is one
// stage's scale chunk for 128 rows (2 KB NVFP4, 512 B MXFP8).
int encode_scale_map(CUtensorMap* map, const void* scales, size_t bytes, uint32_t box_rows) {
    const cuuint64_t dims[2] = {256u, (cuuint64_t)(bytes / 256)};
    const cuuint64_t strides[1] = {256u};
    const cuuint32_t box[2] = {256u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(scales), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVQ_OK : NVQ_ERR_CUDA;
}

// Fields of GemmParams for the quantizing epilogue (EPI 1): MXFP8 codes and
// scales of GELU(D) for an [M, N] output; unused (null) for EPI 0.
void set_epi_quant(GemmParams& p, uint8_t* q_codes, uint8_t* q_sf, int64_t M) {
    p.q_codes = q_codes;
    p.q_sf = q_sf;
    p.m_total = (uint32_t)M;
    p.m_pad = (uint32_t)((M + 127) / 128 * 128);
}

// 256 x BN tiles on CTA pairs (M % 256 == 0, N % BN == 0).  EPI 0 writes D
// (out, ldo); EPI 1 writes MXFP8 codes and scales of GELU(D) (q_codes, q_sf).
template <int FMT, int BN, int EPI>
int launch_gemm_pair(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                     const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                     void* out, int64_t ldo, uint8_t* q_codes, uint8_t* q_sf, int64_t M, int64_t N, int64_t K,
                     cudaStream_t stream) {
    using C = PairCfg<FMT, BN>;
    const int64_t kbytes = FMT == 0 ? K / 2 : K;
    const int fmt = FMT == 0 ? NVQ_NVFP4 : NVQ_MXFP8;   // scale geometry only
    CUtensorMap ma, mb, msa, msb, md;
    memset(&md, 0, sizeof(md));
    int rc;
    if ((rc = encode_codes_map(&ma, a_codes, M, kbytes, 128))) return rc;
    if ((rc = encode_codes_map(&mb, b_codes, N, kbytes, C::BN_HALF))) return rc;
    if ((rc = encode_scale_map(&msa, a_scales, nvq_scale_bytes(fmt, M, K), C::SF_CHUNK / 256))) return rc;
    if ((rc = encode_scale_map(&msb, b_scales, nvq_scale_bytes(fmt, N, K), C::SF_CHUNK / 256))) return rc;
    if (EPI == 0 && (rc = encode_out_map(&md, out, M, N, ldo))) return rc;
    auto kern = bsgemm_pair_kernel<FMT, BN, EPI>;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!d->pair_attr[FMT][BN == 256][EPI]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
                cudaSuccess)
                return NVQ_ERR_CUDA;
            d->pair_attr[FMT][BN == 256][EPI] = true;
        }
    }
    GemmParams p;
    set_epi_quant(p, q_codes, q_sf, M);
    p.sfa = a_scales;
    p.sfb = b_scales;
    p.a_global = a_global;
    p.b_global = b_global;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.status = d->status;
    p.wait_ns = (uint32_t)pipeline_wait_ns(kWaitLimitNs);
    p.num_m_blocks = (uint32_t)((M + 255) / 256);
    p.num_n_blocks = (uint32_t)((N + BN - 1) / BN);
    p.n_total = (uint32_t)N;
    p.sfa_rtiles = (uint32_t)((M + 127) / 128);
    p.sfb_rtiles = (uint32_t)((N + 127) / 128);
    p.num_k_tiles = (uint32_t)(K / C::BK);
    p.sf_ctiles = (uint32_t)(K / C::SF_BLOCK / 4);
    const uint32_t tiles = p.num_m_blocks * p.num_n_blocks;
    const uint32_t pairs = (uint32_t)d->num_sms / 2;
    const uint32_t grid = 2 * (tiles < pairs ? tiles : pairs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, msa, msb, md, p) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

template <int FMT, int BN, int EPI>
int launch_gemm(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                void* out, int64_t ldo, uint8_t* q_codes, uint8_t* q_sf, int64_t M, int64_t N, int64_t K,
                cudaStream_t stream) {
    using C = GemmCfg<FMT, BN>;
    const int64_t kbytes = FMT == 0 ? K / 2 : K;
    CUtensorMap ma, mb, md;
    memset(&md, 0, sizeof(md));
    int rc;
    if ((rc = encode_codes_map(&ma, a_codes, M, kbytes, C::BM))) return rc;
    if ((rc = encode_codes_map(&mb, b_codes, N, kbytes, BN))) return rc;
    if (EPI == 0 && (rc = encode_out_map(&md, out, M, N, ldo))) return rc;
    auto kern = bsgemm_kernel<FMT, BN, EPI>;
    const int wi = BN / 64 - 2;                      // 128 -> 0, 192 -> 1, 256 -> 2
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!d->gemm_attr[FMT][wi][EPI]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
                cudaSuccess)
                return NVQ_ERR_CUDA;
            d->gemm_attr[FMT][wi][EPI] = true;
        }
    }
    GemmParams p;
    set_epi_quant(p, q_codes, q_sf, M);
    p.sfa = a_scales;
    p.sfb = b_scales;
    p.a_global = a_global;
    p.b_global = b_global;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.status = d->status;
    p.wait_ns = (uint32_t)pipeline_wait_ns(kWaitLimitNs);
    p.num_m_blocks = (uint32_t)((M + C::BM - 1) / C::BM);
    p.num_n_blocks = (uint32_t)((N + BN - 1) / BN);
    p.n_total = (uint32_t)N;
    p.sfa_rtiles = (uint32_t)((M + 127) / 128);
    p.sfb_rtiles = (uint32_t)((N + 127) / 128);
    p.num_k_tiles = (uint32_t)(K / C::BK);
    p.sf_ctiles = (uint32_t)(K / C::SF_BLOCK / 4);
    const uint32_t tiles = p.num_m_blocks * p.num_n_blocks;
    const uint32_t grid = tiles < (uint32_t)d->num_sms ? tiles : (uint32_t)d->num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, md, p) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

// Split-K kernel for M <= ROWS: opt in to its shared memory (once per device).
// Call with g_mu held.
template <int FMT, int BN, int ROWS>
bool splitk_opt_in(DeviceInfo* d) {
    bool& done = d->splitk_attr[FMT][BN / 64 - 2][ROWS == 32];
    if (!done) {
        if (cudaFuncSetAttribute(bsgemm_kernel<FMT, BN, 0, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmCfg<FMT, BN, ROWS>::SMEM_BYTES) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        done = true;
    }
    return true;
}

// The number of clusters of `split` split-K CTAs the device holds at once
// (cached; asked of the 32-row kernel, the one with more shared memory).
template <int FMT, int BN>
int splitk_max_clusters(DeviceInfo* d, int split) {
    using C = GemmCfg<FMT, BN, 32>;
    auto kern = bsgemm_kernel<FMT, BN, 0, 32>;
    const int wi = BN / 64 - 2;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!splitk_opt_in<FMT, BN, 32>(d)) return 0;
    int& c = d->splitk_clusters[FMT][wi][split];
    if (c == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(split);
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        c = n + 1;
    }
    return c - 1;
}

// One cluster of `split` CTAs per output tile of M <= ROWS rows and BN
// columns; each CTA sums a contiguous share of the K tiles and the cluster
// adds the partials.  The receive area holds ROWS rows: 16 leaves shared
// memory for more stages than 32.
template <int FMT, int BN, int ROWS>
int launch_gemm_splitk_rows(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                            const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global,
                            const void* bias, void* out, int64_t ldo, int64_t M, int64_t N, int64_t K, int split,
                            cudaStream_t stream) {
    using C = GemmCfg<FMT, BN, ROWS>;
    const int64_t kbytes = FMT == 0 ? K / 2 : K;
    // rows that the receive areas hold, and at least one K tile per CTA of the cluster
    if (M > (int64_t)ROWS || split < 2 || split > 8 || K / C::BK < split) return NVQ_ERR_SHAPE;
    if (splitk_max_clusters<FMT, BN>(d, split) <= 0) return NVQ_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!splitk_opt_in<FMT, BN, ROWS>(d)) return NVQ_ERR_CUDA;
    }
    CUtensorMap ma, mb, md;
    memset(&md, 0, sizeof(md));
    int rc;
    if ((rc = encode_codes_map(&ma, a_codes, M, kbytes, C::A_ROWS))) return rc;
    if ((rc = encode_codes_map(&mb, b_codes, N, kbytes, BN))) return rc;
    GemmParams p;
    set_epi_quant(p, nullptr, nullptr, M);
    p.sfa = a_scales;
    p.sfb = b_scales;
    p.a_global = a_global;
    p.b_global = b_global;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.status = d->status;
    p.wait_ns = (uint32_t)pipeline_wait_ns(kWaitLimitNs);
    p.num_m_blocks = 1;
    p.num_n_blocks = (uint32_t)((N + BN - 1) / BN);
    p.n_total = (uint32_t)N;
    p.sfa_rtiles = 1;
    p.sfb_rtiles = (uint32_t)((N + 127) / 128);
    p.num_k_tiles = (uint32_t)(K / C::BK);
    p.sf_ctiles = (uint32_t)(K / C::SF_BLOCK / 4);
    p.k_split = (uint32_t)split;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.ldo = (uint32_t)ldo;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.num_n_blocks * (uint32_t)split);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = split;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, bsgemm_kernel<FMT, BN, 0, ROWS>, ma, mb, md, p) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

template <int FMT, int BN>
int launch_gemm_splitk(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                       const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                       void* out, int64_t ldo, int64_t M, int64_t N, int64_t K, int split, cudaStream_t stream) {
    if (M <= 16)
        return launch_gemm_splitk_rows<FMT, BN, 16>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global,
                                                    bias, out, ldo, M, N, K, split, stream);
    return launch_gemm_splitk_rows<FMT, BN, 32>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                                out, ldo, M, N, K, split, stream);
}

// Fused short-M NVFP4 linear: one cluster of `split` CTAs per 16 x BN output
// tile, the activation quantized inside the kernel (fused_quantize_a).
// Needs every CTA's share of the K tiles to fit its stages at once.
template <int BN>
int launch_linear_short(DeviceInfo* d, const void* x, int64_t ldx, const uint8_t* b_codes, const uint8_t* b_scales,
                        const float* b_global, const void* bias, void* out, int64_t ldo, uint8_t* a_codes,
                        uint8_t* a_scales, float* a_global, int64_t M, int64_t N, int64_t K, int split,
                        cudaStream_t stream) {
    using C = GemmCfg<0, BN, 16, true>;
    auto kern = bsgemm_kernel<0, BN, 0, 16, true>;
    const int64_t nkt = K / C::BK;
    if (M > 16 || split < 2 || split > 8 || nkt < split || (nkt + split - 1) / split > C::STAGES)
        return NVQ_ERR_SHAPE;
    if (splitk_max_clusters<0, BN>(d, split) <= 0) return NVQ_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        bool& done = d->short_attr[BN / 64 - 2];
        if (!done) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
                cudaSuccess) {
                cudaGetLastError();
                return NVQ_ERR_CUDA;
            }
            done = true;
        }
    }
    CUtensorMap mb, md;
    memset(&md, 0, sizeof(md));
    int rc;
    if ((rc = encode_codes_map(&mb, b_codes, N, K / 2, BN))) return rc;
    GemmParams p;
    set_epi_quant(p, a_codes, a_scales, M);
    p.ldx = (uint32_t)ldx;
    p.x = static_cast<const uint16_t*>(x);
    p.sfb = b_scales;
    p.a_global_out = a_global;
    p.b_global = b_global;
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.status = d->status;
    p.wait_ns = (uint32_t)pipeline_wait_ns(kWaitLimitNs);
    p.num_m_blocks = 1;
    p.num_n_blocks = (uint32_t)((N + BN - 1) / BN);
    p.n_total = (uint32_t)N;
    p.sfa_rtiles = 1;
    p.sfb_rtiles = (uint32_t)((N + 127) / 128);
    p.num_k_tiles = (uint32_t)nkt;
    p.sf_ctiles = (uint32_t)(K / C::SF_BLOCK / 4);
    p.k_split = (uint32_t)split;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.ldo = (uint32_t)ldo;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.num_n_blocks * (uint32_t)split);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = split;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // tmap_a is not read on this path; the B map stands in for it
    if (cudaLaunchKernelEx(&cfg, kern, mb, mb, md, p) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

struct GemmPlan {
    int tile_m, tile_n, k_split;
};

// The kernel block_scaled_linear runs for a shape.  CTA pairs (256-row
// tiles) unless M fits one 128-row tile: 256 x 256 tiles, or 256 x 192 (two
// accumulators for MXFP8) when N is a multiple of 384 but not of 256.
// Measured on the FF-up shape, 256 x 256 with one accumulator is faster than
// 256 x 192 with two.  A ragged N takes 256.  One CTA per tile otherwise:
// width 256 when N allows it (fewest scale-factor copies per MMA), else 192,
// else 128 (two accumulators); when 256-wide tiles would leave SMs idle (a
// short M: the weight stream is then the cost), 128-wide tiles spread it over
// twice as many SMs.  At M <= kSplitKMaxRows, K is split across a cluster when that
// streams the weight through at least a quarter more SMs than the best
// unsplit grid: the tile width (256, 192 or 128) and split that occupy the
// most SMs in one wave of clusters (at least two K tiles per CTA, at most 8
// CTAs per cluster, and no more clusters than the device holds at once: on
// a B200 that is 74 clusters of 2 but only 45 of 3), the wider tile and then
// the smaller split on a tie.
// Rows up to which a K split pays, which are also the rows the split
// kernel's receive areas hold.  The exchange grows with M: with partials
// read back through distributed shared memory, the split kernel measured
// 9.2 / 10.1 / 10.1 / 10.3 / 11.6 us on the FF-up weight at M = 1 / 16 / 32
// / 64 / 128 against 10.8 / 10.9 / 10.7 / 9.8 / 9.4 us unsplit.
constexpr int64_t kSplitKMaxRows = kSplitKRows;

// The plan as a function of the shape and of the device's facts: its SM
// count and fit(w, sp), the most clusters of sp CTAs with w-wide tiles that
// it holds at once.  bk = K elements per pipeline stage.
template <typename Fit>
GemmPlan plan_gemm_core(int64_t bk, int64_t M, int64_t N, int64_t K, int num_sms, bool pairs, bool splitk,
                        Fit fit) {
    if (pairs && M > 128) return {256, (N % 384 == 0 && N % 256 != 0) ? 192 : 256, 1};
    int bn = 128;
    if ((M + 127) / 128 * ((N + 255) / 256) >= num_sms) bn = N % 256 == 0 ? 256 : N % 384 == 0 ? 192 : 128;
    GemmPlan plan = {128, bn, 1};
    if (!splitk || M > kSplitKMaxRows) return plan;
    const int64_t nkt = K / bk;
    const int64_t base = (N + bn - 1) / bn;
    int64_t best = base;
    GemmPlan split = plan;
    for (int w : {256, 192, 128}) {
        const int64_t tiles = (N + w - 1) / w;
        for (int sp = 2; sp <= 8 && 2 * sp <= nkt && tiles * sp <= num_sms; ++sp) {
            if (tiles * sp <= best) continue;
            if (tiles > fit(w, sp)) continue;
            best = tiles * sp;
            split = {128, w, sp};
        }
    }
    return best * 4 >= base * 5 ? split : plan;
}

template <int FMT>
GemmPlan plan_gemm(DeviceInfo* d, int64_t M, int64_t N, int64_t K) {
    return plan_gemm_core(GemmCfg<FMT, 128>::BK, M, N, K, d->num_sms, g_use_pairs, g_use_splitk,
                          [d](int w, int sp) {
                              return w == 256   ? splitk_max_clusters<FMT, 256>(d, sp)
                                     : w == 192 ? splitk_max_clusters<FMT, 192>(d, sp)
                                                : splitk_max_clusters<FMT, 128>(d, sp);
                          });
}

}  // namespace
// One launch per (format, tile shape); FMT 0 = NVFP4, 1 = MXFP8 (E4M3), 2 = MXFP8 (E5M2).
template <int FMT>
int launch_for_format(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                      const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                      void* out, int64_t ldo, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
    const GemmPlan pl = plan_gemm<FMT>(d, M, N, K);
    if (pl.tile_m == 256) {
        if (pl.tile_n == 192)
            return launch_gemm_pair<FMT, 192, 0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                                 out, ldo, nullptr, nullptr, M, N, K, s);
        return launch_gemm_pair<FMT, 256, 0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                             out, ldo, nullptr, nullptr, M, N, K, s);
    }
    if (pl.k_split > 1) {
        if (pl.tile_n == 256)
            return launch_gemm_splitk<FMT, 256>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                                out, ldo, M, N, K, pl.k_split, s);
        if (pl.tile_n == 192)
            return launch_gemm_splitk<FMT, 192>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                                out, ldo, M, N, K, pl.k_split, s);
        return launch_gemm_splitk<FMT, 128>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out,
                                            ldo, M, N, K, pl.k_split, s);
    }
    if (pl.tile_n == 256)
        return launch_gemm<FMT, 256, 0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out, ldo,
                                        nullptr, nullptr, M, N, K, s);
    if (pl.tile_n == 192)
        return launch_gemm<FMT, 192, 0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out, ldo,
                                        nullptr, nullptr, M, N, K, s);
    return launch_gemm<FMT, 128, 0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out, ldo,
                                    nullptr, nullptr, M, N, K, s);
}

// The quantizing epilogue (GELU, then MXFP8 codes and scales) on 256-wide
// tiles: CTA pairs as above, else one CTA per 128 x 256 tile, or 128 x 128
// when 256-wide tiles would leave SMs idle.
template <int FMT>
int launch_gelu_mxfp8(DeviceInfo* d, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                      const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                      uint8_t* y_codes, uint8_t* y_scales, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
    if (g_use_pairs && M > 128)
        return launch_gemm_pair<FMT, 256, 1>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias,
                                             nullptr, 0, y_codes, y_scales, M, N, K, s);
    if ((M + 127) / 128 * ((N + 255) / 256) < d->num_sms)
        return launch_gemm<FMT, 128, 1>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, nullptr,
                                        0, y_codes, y_scales, M, N, K, s);
    return launch_gemm<FMT, 256, 1>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, nullptr, 0,
                                    y_codes, y_scales, M, N, K, s);
}

}  // namespace nvq

using namespace nvq;

extern "C" {

size_t nvq_codes_bytes(int format, int64_t rows, int64_t K) {
    if ((format != NVQ_NVFP4 && !is_mxfp8(format)) || rows < 0 || K < 0) return 0;
    return (size_t)(format == NVQ_NVFP4 ? rows * (K / 2) : rows * K);
}

size_t nvq_scale_bytes(int format, int64_t rows, int64_t K) {
    if ((format != NVQ_NVFP4 && !is_mxfp8(format)) || rows < 0 || K < 0) return 0;
    const int64_t cols = K / block_of(format);
    return (size_t)(((rows + 127) / 128) * 128 * ((cols + 3) / 4) * 4);
}

size_t nvq_workspace_bytes(void) { return kWorkspaceBytes; }

int nvfp4_quantize(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                   float* global_scale, const float* calib_amax, void* workspace, nvq_stream_t stream) {
    return nvfp4_quantize_impl(x, M, K, ldx, codes, scales, global_scale, calib_amax, workspace,
                               reinterpret_cast<cudaStream_t>(stream));
}

int mxfp8_quantize(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                   nvq_stream_t stream) {
    return mxfp8_quantize_impl(x, M, K, ldx, codes, scales, NVQ_MXFP8, NVQ_SCALE_FLOOR,
                               reinterpret_cast<cudaStream_t>(stream));
}

int mxfp8_quantize_ex(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                      int elem_format, int scale_rule, nvq_stream_t stream) {
    return mxfp8_quantize_impl(x, M, K, ldx, codes, scales, elem_format, scale_rule,
                               reinterpret_cast<cudaStream_t>(stream));
}

int quantize_weight(int format, const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* codes,
                    uint8_t* scales, float* global_scale, void* workspace, nvq_stream_t stream) {
    if (format == NVQ_NVFP4)
        return nvfp4_quantize_impl(w, N, K, ldw, codes, scales, global_scale, nullptr, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
    if (is_mxfp8(format))
        return mxfp8_quantize_impl(w, N, K, ldw, codes, scales, format, NVQ_SCALE_FLOOR,
                                   reinterpret_cast<cudaStream_t>(stream));
    return NVQ_ERR_FORMAT;
}

int nvfp4_linear_short_m(const void* x, int64_t M, int64_t K, int64_t ldx, const uint8_t* b_codes,
                         const uint8_t* b_scales, const float* b_global, const void* bias, void* out, int64_t ldo,
                         int64_t N, uint8_t* a_codes, uint8_t* a_scales, float* a_global, nvq_stream_t stream) {
    int rc = check_quant_shape(NVQ_NVFP4, M, K, ldx);
    if (rc) return rc;
    if (M > 16 || N <= 0 || N % 8 || K % 256) return NVQ_ERR_SHAPE;
    if (ldo < N || ldo % 8 || ldo >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    if (M == 0) return NVQ_OK;
    if (!x || !b_codes || !b_scales || !b_global || !out) return NVQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(out) ||
        (a_codes && !aligned16(a_codes)) || (a_scales && !aligned16(a_scales)) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) || (a_global && (reinterpret_cast<uintptr_t>(a_global) & 3u)))
        return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d))) return rc;
    if ((rc = get_encoder())) return rc;
    const GemmPlan pl = plan_gemm<0>(d, M, N, K);
    if (pl.k_split < 2) return NVQ_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (pl.tile_n == 256)
        return launch_linear_short<256>(d, x, ldx, b_codes, b_scales, b_global, bias, out, ldo, a_codes, a_scales,
                                        a_global, M, N, K, pl.k_split, s);
    if (pl.tile_n == 192)
        return launch_linear_short<192>(d, x, ldx, b_codes, b_scales, b_global, bias, out, ldo, a_codes, a_scales,
                                        a_global, M, N, K, pl.k_split, s);
    return launch_linear_short<128>(d, x, ldx, b_codes, b_scales, b_global, bias, out, ldo, a_codes, a_scales,
                                    a_global, M, N, K, pl.k_split, s);
}

int block_scaled_linear(int format, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, const void* bias,
                        void* out, int64_t ldo, int64_t M, int64_t N, int64_t K, nvq_stream_t stream) {
    if (format != NVQ_NVFP4 && !is_mxfp8(format)) return NVQ_ERR_FORMAT;
    // the GEMM stages 256 (NVFP4) / 128 (MXFP8) elements of K at a time;
    // M and N may be ragged (tensor-map loads fill past the end with zeros,
    // stores are clipped)
    const int64_t k_stage = format == NVQ_NVFP4 ? 256 : 128;
    // N a multiple of 8: the tensor-map store of the last column chunk clips
    // at 16-byte granularity, so a BF16 row must end on a 16-byte boundary
    if (M < 0 || N <= 0 || N % 8 || K <= 0 || K % k_stage) return NVQ_ERR_SHAPE;
    if (ldo < N || ldo % 8 || M * ldo >= (int64_t(1) << 40) || ldo >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    if (K >= (int64_t(1) << 24) || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    if (M == 0) return NVQ_OK;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !out) return NVQ_ERR_NULL;
    if (format == NVQ_NVFP4 && (!a_global || !b_global)) return NVQ_ERR_NULL;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
        !aligned16(out) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    if ((rc = get_encoder())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (format == NVQ_NVFP4)
        return launch_for_format<0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, out, ldo, M, N,
                                    K, s);
    if (format == NVQ_MXFP8)
        return launch_for_format<1>(d, a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, bias, out, ldo, M, N,
                                    K, s);
    return launch_for_format<2>(d, a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, bias, out, ldo, M, N, K,
                                s);
}

namespace {
int check_plan_args(int format, int64_t M, int64_t N, int64_t K, const int* tile_m, const int* tile_n,
                    const int* k_split) {
    if (format != NVQ_NVFP4 && !is_mxfp8(format)) return NVQ_ERR_FORMAT;
    if (!tile_m || !tile_n || !k_split) return NVQ_ERR_NULL;
    const int64_t k_stage = format == NVQ_NVFP4 ? 256 : 128;
    if (M <= 0 || N <= 0 || N % 8 || K <= 0 || K % k_stage) return NVQ_ERR_SHAPE;
    if (K >= (int64_t(1) << 24) || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    return NVQ_OK;
}
}  // namespace

int nvq_gemm_plan_host(int format, int64_t M, int64_t N, int64_t K, int num_sms, const int* max_clusters,
                       int use_pairs, int use_splitk, int* tile_m, int* tile_n, int* k_split) {
    int rc = check_plan_args(format, M, N, K, tile_m, tile_n, k_split);
    if (rc) return rc;
    if (!max_clusters) return NVQ_ERR_NULL;
    if (num_sms <= 0) return NVQ_ERR_SHAPE;
    const int64_t bk = format == NVQ_NVFP4 ? 256 : 128;
    const GemmPlan pl = plan_gemm_core(bk, M, N, K, num_sms, use_pairs != 0, use_splitk != 0,
                                       [max_clusters](int w, int sp) { return max_clusters[(w / 64 - 2) * 9 + sp]; });
    *tile_m = pl.tile_m;
    *tile_n = pl.tile_n;
    *k_split = pl.k_split;
    return NVQ_OK;
}

int nvq_gemm_plan(int format, int64_t M, int64_t N, int64_t K, int* tile_m, int* tile_n, int* k_split) {
    int rc = check_plan_args(format, M, N, K, tile_m, tile_n, k_split);
    if (rc) return rc;
    DeviceInfo* d = nullptr;
    rc = device_info(&d);
    if (rc) return rc;
    const GemmPlan pl = format == NVQ_NVFP4 ? plan_gemm<0>(d, M, N, K)
                        : format == NVQ_MXFP8 ? plan_gemm<1>(d, M, N, K)
                                              : plan_gemm<2>(d, M, N, K);
    *tile_m = pl.tile_m;
    *tile_n = pl.tile_n;
    *k_split = pl.k_split;
    return NVQ_OK;
}

int block_scaled_linear_gelu_mxfp8(int format, const uint8_t* a_codes, const uint8_t* a_scales,
                                   const float* a_global, const uint8_t* b_codes, const uint8_t* b_scales,
                                   const float* b_global, const void* bias, uint8_t* y_codes, uint8_t* y_scales,
                                   int64_t M, int64_t N, int64_t K, nvq_stream_t stream) {
    if (format != NVQ_NVFP4 && format != NVQ_MXFP8) return NVQ_ERR_FORMAT;
    const int64_t k_stage = format == NVQ_NVFP4 ? 256 : 128;
    // N is the K of the next layer's MXFP8 operand: whole 4-block scale columns
    if (M < 0 || N <= 0 || N % 128 || K <= 0 || K % k_stage) return NVQ_ERR_SHAPE;
    if (K >= (int64_t(1) << 24) || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) ||
        M * N >= (int64_t(1) << 40))
        return NVQ_ERR_SHAPE;
    if (M == 0) return NVQ_OK;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !y_codes || !y_scales) return NVQ_ERR_NULL;
    if (format == NVQ_NVFP4 && (!a_global || !b_global)) return NVQ_ERR_NULL;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
        !aligned16(y_codes) || !aligned16(y_scales) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    if ((rc = get_encoder())) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (format == NVQ_NVFP4)
        return launch_gelu_mxfp8<0>(d, a_codes, a_scales, a_global, b_codes, b_scales, b_global, bias, y_codes,
                                    y_scales, M, N, K, s);
    return launch_gelu_mxfp8<1>(d, a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, bias, y_codes, y_scales,
                                M, N, K, s);
}

int nvq_probe_gelu(const uint16_t* in, int64_t n, uint16_t* out, nvq_stream_t stream) {
    if (!in || !out) return NVQ_ERR_NULL;
    if (n < 0 || n >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    if (n == 0) return NVQ_OK;
    uint64_t grid = ((uint64_t)n + 255) / 256;
    if (grid > (uint64_t)d->num_sms) grid = (uint64_t)d->num_sms;
    probe_gelu_kernel<<<(uint32_t)grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, (uint32_t)n, out);
    return launch_status();
}

int nvq_probe_wait(uint64_t limit_ns, unsigned long long* waited_ns, nvq_stream_t stream) {
    if (!waited_ns) return NVQ_ERR_NULL;
    if (limit_ns > 1000000000ull) return NVQ_ERR_SHAPE;    // at most 1 s
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    probe_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, d->status, waited_ns);
    return launch_status();
}

int nvq_debug_build(void) { return kDebugBuild ? 1 : 0; }

int nvq_probe_bounds(nvq_stream_t stream) {
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    probe_bounds_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d->status);
    return launch_status();
}

int nvq_set_wait_limit(uint64_t limit_ns) {
    if (limit_ns > kWaitLimitNs) return NVQ_ERR_SHAPE;       // at most the 4 s default
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    return NVQ_OK;
}

uint64_t nvq_wait_limit(void) { return g_wait_limit_ns.load(std::memory_order_relaxed); }

int nvq_workspace_init(void* workspace, nvq_stream_t stream) {
    if (!workspace) return NVQ_ERR_NULL;
    if (!aligned16(workspace)) return NVQ_ERR_ALIGN;
    if (cudaMemsetAsync(workspace, 0, kWorkspaceBytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return NVQ_ERR_CUDA;
    }
    return NVQ_OK;
}

int nvq_device_status(nvq_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NVQ_ERR_CUDA;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    unsigned int v = 0;
    if (cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return NVQ_ERR_CUDA;
    const unsigned int zero = 0;
    if (cudaMemcpy(d->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return NVQ_ERR_CUDA;
    return (int)v;
}

const char* nvq_status_string(int code) {
    switch (code) {
        case NVQ_OK: return "ok";
        case NVQ_ERR_NULL: return "null pointer";
        case NVQ_ERR_SHAPE: return "shape or pitch breaks the contract";
        case NVQ_ERR_ALIGN: return "pointer not 16-byte aligned";
        case NVQ_ERR_ARCH: return "device is not compute capability 10.0 (sm_100a)";
        case NVQ_ERR_CUDA: return "CUDA error";
        case NVQ_ERR_FORMAT: return "unknown format";
        default: return "unknown status";
    }
}

int nvq_probe_convert(const float* in, int64_t n, uint8_t* e2m1_out, uint8_t* e4m3_out, nvq_stream_t stream) {
    if (!in || !e2m1_out || !e4m3_out) return NVQ_ERR_NULL;
    if (n < 0 || n >= (int64_t(1) << 31)) return NVQ_ERR_SHAPE;
    DeviceInfo* d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    if (n == 0) return NVQ_OK;
    const uint32_t grid = quant_grid((uint64_t)n, d->num_sms);
    probe_convert_kernel<<<grid, kQuantThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        in, (uint32_t)n, e2m1_out, e4m3_out);
    return launch_status();
}

int nvfp4_quantize_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* scales,
                           float* global_scale, nvq_stream_t stream) {
    // Device address of the static scratch array, looked up on this entry
    // point's first call on each device (with that device current).
    static uint32_t* scratch[kMaxDevices] = {};
    int rc = check_quant_shape(NVQ_NVFP4, M, K, ldx);
    if (rc) return rc;
    if (M == 0) return NVQ_OK;
    if (!x || !codes || !scales || !global_scale) return NVQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return NVQ_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(global_scale) & 3u) return NVQ_ERR_ALIGN;
    DeviceInfo* d = nullptr;
    if ((rc = device_info(&d))) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVQ_ERR_CUDA;
    uint32_t* partials = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!scratch[dev]) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_partials) != cudaSuccess) return NVQ_ERR_CUDA;
            scratch[dev] = static_cast<uint32_t*>(ptr);
        }
        partials = scratch[dev];
    }
    // the amax pass writes one partial per CTA and launches at most as many
    // CTAs as the static scratch holds
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t npartial = 0;
    if ((rc = launch_amax(x, M, K, ldx, partials, NVQ_NOALLOC_MAX_PARTIALS, d->num_sms, d->status, s, &npartial))) return rc;
    const uint32_t nblk = (uint32_t)(K / 16);
    const float* no_calib = nullptr;
    return launch_pdl(nvfp4_quantize_kernel, dim3(quant_grid((uint64_t)M * nblk, d->num_sms)), dim3(kQuantThreads), 0,
                      s, static_cast<const uint16_t*>(x), (uint32_t)M, nblk, (uint32_t)ldx, codes, scales,
                      global_scale, partials, npartial, no_calib, d->status);
}

}  // extern "C"
