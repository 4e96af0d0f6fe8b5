// qlora_api.cu -- the C ABI of libqlora.so (declared in include/qlora.h):
// argument validation, workspace layout, tensor-map encoding and the launch
// sequence of each call.  No device memory is allocated here.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <atomic>
#include <mutex>
#include <set>
#include <string>
#include <utility>

#include "../../include/qlora.h"
#include "internal.h"
#include "ptx.cuh"
#include "tile_epilogue.cuh"

namespace qlora {

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

// Device status word (one per device context): kernels record a timed-out
// bounded wait here; qlora_device_status() reads and clears it.
__device__ int g_device_status;

std::mutex g_mu;
int* g_status_ptr[64] = {nullptr};

int* status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Forward: Xq [M,K] int8 and sx [M] fp32.  Backward: the G slices
// Gp [ncb][M,r] fp32 (written by the dY pass, read by the dX GEMM and the X
// pass) and, when there are more than kMaxDirectSlices slices, their sum
// G [M,r].  The two uses do not overlap in time.
struct WsLayout {
    size_t xq, sx, fwd_total;
    size_t gp, g, bwd_total;
    int ncb;
    bool reduce;  // consumers read G (added once) instead of the slices
    size_t total;
};

WsLayout layout_for(const qlora_layer_desc& d, int M) {
    WsLayout w{};
    const Act act = d.act_dtype == QLORA_BF16 ? kBF16 : kF32;
    w.xq = 0;
    w.sx = align256(static_cast<size_t>(M) * d.K);
    w.fwd_total = w.sx + align256(static_cast<size_t>(M) * 4);
    w.ncb = rank_col_blocks(act, d.N);
    w.reduce = w.ncb > kMaxDirectSlices;
    w.gp = 0;
    w.g = align256(static_cast<size_t>(w.ncb) * M * d.r * 4);
    w.bwd_total = w.g + (w.reduce ? align256(static_cast<size_t>(M) * d.r * 4) : 0);
    w.total = w.fwd_total > w.bwd_total ? w.fwd_total : w.bwd_total;
    return w;
}

// Where the consumers read G: the slices themselves, or G once added up.
const float* g_source(const WsLayout& w, const void* ws, int* nsl) {
    const uint8_t* b = static_cast<const uint8_t*>(ws);
    *nsl = w.reduce ? 1 : w.ncb;
    return reinterpret_cast<const float*>(b + (w.reduce ? w.g : w.gp));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_desc(const qlora_layer_desc* d) {
    if (!d) return fail(QLORA_EINVAL, "layer descriptor is NULL");
    if (d->K < 1 || d->N < 1) return fail(QLORA_ESHAPE, "K and N must be >= 1");
    if (d->r < 1 || d->r > 64) return fail(QLORA_ESHAPE, "rank r must be in [1, 64]");
    if (d->K % 16 != 0)
        return fail(QLORA_EUNSUPPORTED, "K must be a multiple of 16 (16-byte int8 row pitch)");
    if (d->K > 131072)
        return fail(QLORA_EUNSUPPORTED, "K > 131072 would overflow the int32 accumulator");
    if (d->act_dtype != QLORA_F32 && d->act_dtype != QLORA_BF16)
        return fail(QLORA_EINVAL, "unknown activation dtype");
    return QLORA_OK;
}

int cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return QLORA_OK;
    return fail(QLORA_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t rows, uint64_t cols, uint64_t pitch_bytes, uint32_t box_rows,
                  uint32_t box_cols, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    (void)elem_bytes;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d_blocks(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, uint64_t rows, uint64_t cols, uint32_t blk,
                         uint32_t box_rows, uint32_t box_blocks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || cols % blk != 0) return false;
    const uint64_t eb = static_cast<uint64_t>(elem_bytes);
    cuuint64_t dims[3] = {blk, rows, cols / blk};
    cuuint64_t strides[2] = {cols * eb, blk * eb};
    cuuint32_t box[3] = {blk, box_rows, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
std::atomic<int> g_rank_pass_rows{0};
}

int rank_pass_rows() { return g_rank_pass_rows.load(std::memory_order_relaxed); }

int sm_count() {
    // per device, looked up once (0: not yet); racing first lookups store the same value
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

int greatest_priority() {
    // per device, looked up once; threads that race on the first lookup
    // store the same value
    static std::atomic<int> cache[64] = {};
    static std::atomic<bool> init[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!init[dev].load(std::memory_order_acquire)) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
        cache[dev].store(greatest, std::memory_order_relaxed);
        init[dev].store(true, std::memory_order_release);
    }
    return cache[dev].load(std::memory_order_relaxed);
}

cudaError_t ensure_smem_attr(const void* func, int bytes) {
    // largest dynamic shared memory size set so far, per (device, kernel):
    // some kernels size their shared memory by the rank at run time
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, int> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    auto it = done.find({dev, func});
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[{dev, func}] = bytes;
    return e;
}

}  // namespace qlora

namespace qlora {
namespace {

// Scratch of qlora_backward_noalloc: the G slices of the rank-r backward live
// in this file-scope array (one copy per device, reserved when the module is
// loaded on that device) instead of a caller-supplied workspace.  Every
// element the three passes read is written by the dY pass of the same call
// first, so nothing in it has to start at zero.
__device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

uint8_t* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t noalloc_scratch(uint8_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_version(void) { return "qlora-b200 0.1 sm_100a"; }

const char* qlora_last_error(void) { return g_last_error.c_str(); }

int qlora_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "stream synchronisation failed");
    int* p = status_ptr();
    if (!p) return fail(QLORA_ECUDA, "device status word unavailable");
    int v = 0;
    e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "reading the device status word");
    if (v != 0) {
        int zero = 0;
        cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
        return fail(QLORA_ETIMEOUT, "a kernel gave up a bounded wait");
    }
    return QLORA_OK;
}

size_t qlora_workspace_bytes(const qlora_layer_desc* d, int M) {
    if (check_desc(d) != QLORA_OK || M < 0) return 0;
    if (M == 0) return 256;
    return layout_for(*d, M).total;
}

int qlora_quantize_weight(const float* W, int K, int N, int8_t* Wq, float* sw, void* stream) {
    if (!W || !Wq || !sw) return fail(QLORA_EINVAL, "NULL pointer argument");
    if (K < 1 || N < 1) return fail(QLORA_ESHAPE, "K and N must be >= 1");
    if (K % 16 != 0) return fail(QLORA_EUNSUPPORTED, "K must be a multiple of 16");
    if (!aligned(W, 4) || !aligned(sw, 4) || !aligned(Wq, 16))
        return fail(QLORA_EALIGN, "misaligned pointer (W, sw 4 B; Wq 16 B)");
    return cuda_status(launch_quantize_weight(W, K, N, Wq, sw, static_cast<cudaStream_t>(stream)),
                       "quantize_weight launch");
}

// ---------------------------------------------------------------------------
// step-level entry points (a1 .. a5) and their compositions
// ---------------------------------------------------------------------------
#define QL_REQUIRE(cond, code, msg) \
    do {                            \
        if (!(cond)) return fail((code), (msg)); \
    } while (0)

static int check_layer(const qlora_layer_desc* d, int M) {
    int rc = check_desc(d);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(M >= 0, QLORA_ESHAPE, "M must be >= 0");
    return QLORA_OK;
}

static Act act_of(const qlora_layer_desc* d) { return d->act_dtype == QLORA_BF16 ? kBF16 : kF32; }
static float lora_scale(const qlora_layer_desc* d) { return d->alpha / static_cast<float>(d->r); }

int qlora_quantize_input(const qlora_layer_desc* d, int M, const void* X, const float* A,
                         int8_t* Xq, float* sx, float* xA, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && A && Xq && sx && xA, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(X, 16) && aligned(Xq, 16), QLORA_EALIGN, "X and Xq must be 16-byte aligned");
    QL_REQUIRE(aligned(A, 4) && aligned(sx, 4) && aligned(xA, 4), QLORA_EALIGN,
               "fp32 vectors must be 4-byte aligned");
    if (M == 0) return QLORA_OK;
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    return cuda_status(launch_quantize_rows(act_of(d), X, A, M, d->K, d->r, Xq, sx, xA, status,
                                            static_cast<cudaStream_t>(stream)),
                       "input quantizer launch");
}

static int gemm_forward_impl(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                             const int8_t* Wq, const float* sw, const float* bias,
                             const float* xA, const float* B, void* Y, int32_t* acc, int relu,
                             void* stream, bool w4 = false) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(!w4 || d->K % 32 == 0, QLORA_EUNSUPPORTED,
               "packed int4 kernels need K a multiple of 32 (16-byte rows of codes)");
    QL_REQUIRE(Xq && sx && Wq && sw && xA && B && Y, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(Xq, 16) && aligned(Wq, 16) && aligned(Y, 16), QLORA_EALIGN,
               "Xq, Wq and Y must be 16-byte aligned");
    QL_REQUIRE(aligned(sx, 4) && aligned(sw, 4) && aligned(xA, 4) && aligned(B, 4) &&
                   (!bias || aligned(bias, 4)) && (!acc || aligned(acc, 4)),
               QLORA_EALIGN, "fp32/int32 vectors must be 4-byte aligned");
    if (M == 0) return QLORA_OK;
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    FwdEpilogue ep;
    ep.sx = sx;
    ep.sw = sw;
    ep.bias = bias;
    ep.xA = xA;
    ep.B = B;
    ep.r = d->r;
    ep.c = lora_scale(d);
    ep.Y = Y;
    ep.acc = acc;
    ep.relu = relu;
    return cuda_status(launch_gemm_i8_fwd(act_of(d), Xq, Wq, M, d->N, d->K, ep, status,
                                          static_cast<cudaStream_t>(stream), w4),
                       "int8 GEMM launch");
}

int qlora_gemm_forward(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                       const int8_t* Wq, const float* sw, const float* bias, const float* xA,
                       const float* B, void* Y, int32_t* acc, void* stream) {
    return gemm_forward_impl(d, M, Xq, sx, Wq, sw, bias, xA, B, Y, acc, 0, stream);
}

int qlora_gemm_forward_relu(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                            const int8_t* Wq, const float* sw, const float* bias, const float* xA,
                            const float* B, void* Y, int32_t* acc, void* stream) {
    return gemm_forward_impl(d, M, Xq, sx, Wq, sw, bias, xA, B, Y, acc, 1, stream);
}

int qlora_lora_grad_dy(const qlora_layer_desc* d, int M, const void* dY, const float* B,
                       const float* xA, float* dB, float* dbias, float* G, void* workspace,
                       size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(dY && B && xA && dB && workspace, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(dY, 16) && aligned(workspace, 256), QLORA_EALIGN,
               "dY must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(B, 4) && aligned(xA, 4) && (!G || aligned(G, 4)) && aligned(dB, 4) &&
                   (!dbias || aligned(dbias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        rc = cuda_status(cudaMemsetAsync(dB, 0, sizeof(float) * d->r * d->N, s), "memset dB");
        if (rc == QLORA_OK && dbias)
            rc = cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * d->N, s), "memset dbias");
        return rc;
    }
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    float* gp = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.gp);
    rc = cuda_status(launch_rank_dy(act_of(d), dY, B, xA, M, d->N, d->r, lora_scale(d), gp, dB,
                                    dbias, status, s),
                     "dY pass launch");
    if (rc == QLORA_OK && w.reduce)
        rc = cuda_status(launch_g_reduce(gp, w.ncb, M, d->r,
                                         reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.g),
                                         s),
                         "G reduction launch");
    if (rc == QLORA_OK && G)
        rc = cuda_status(launch_g_reduce(gp, w.ncb, M, d->r, G, s), "G reduction launch");
    return rc;
}

int qlora_lora_g(const qlora_layer_desc* d, int M, const void* dY, const float* B,
                 void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(dY && B && workspace, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(dY, 16) && aligned(workspace, 256), QLORA_EALIGN,
               "dY must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(B, 4), QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    if (M == 0) return QLORA_OK;
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* gp = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.gp);
    rc = cuda_status(launch_rank_dy(act_of(d), dY, B, nullptr, M, d->N, d->r, lora_scale(d), gp,
                                    nullptr, nullptr, status, s),
                     "G pass launch");
    if (rc == QLORA_OK && w.reduce)
        rc = cuda_status(launch_g_reduce(gp, w.ncb, M, d->r,
                                         reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.g),
                                         s),
                         "G reduction launch");
    return rc;
}

int qlora_lora_grad_b(const qlora_layer_desc* d, int M, const void* dY, const float* xA,
                      float* dB, float* dbias, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(dY && xA && dB, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(dY, 16), QLORA_EALIGN, "dY must be 16-byte aligned");
    QL_REQUIRE(aligned(xA, 4) && aligned(dB, 4) && (!dbias || aligned(dbias, 4)), QLORA_EALIGN,
               "fp32 vectors must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        rc = cuda_status(cudaMemsetAsync(dB, 0, sizeof(float) * d->r * d->N, s), "memset dB");
        if (rc == QLORA_OK && dbias)
            rc = cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * d->N, s), "memset dbias");
        return rc;
    }
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    return cuda_status(launch_rank_dy(act_of(d), dY, nullptr, xA, M, d->N, d->r, lora_scale(d),
                                      nullptr, dB, dbias, status, s),
                       "dB pass launch");
}

static int gemm_dx_impl(const qlora_layer_desc* d, int M, const void* dY, const int8_t* Wq,
                        const float* sw, const float* A, const void* gate, void* dX,
                        const void* workspace, size_t workspace_bytes, void* stream,
                        bool w4 = false) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(!w4 || d->K % 32 == 0, QLORA_EUNSUPPORTED,
               "packed int4 kernels need K a multiple of 32 (16-byte rows of codes)");
    QL_REQUIRE(dY && Wq && sw && A && dX && workspace, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(dY, 16) && aligned(Wq, 16) && aligned(dX, 16) && aligned(workspace, 256),
               QLORA_EALIGN, "dY, Wq and dX must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(sw, 4) && aligned(A, 4), QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    QL_REQUIRE(!gate || aligned(gate, 16), QLORA_EALIGN, "X must be 16-byte aligned");
    if (M == 0) return QLORA_OK;
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    DxEpilogue ep;
    ep.Gp = g_source(w, workspace, &ep.ncb);
    ep.A = A;
    ep.r = d->r;
    ep.c = lora_scale(d);
    ep.dX = dX;
    ep.gate = gate;
    return cuda_status(launch_gemm_dx(act_of(d), dY, Wq, sw, M, d->N, d->K, ep, status,
                                      static_cast<cudaStream_t>(stream), w4),
                       "dX GEMM launch");
}

int qlora_gemm_dx(const qlora_layer_desc* d, int M, const void* dY, const int8_t* Wq,
                  const float* sw, const float* A, void* dX, const void* workspace,
                  size_t workspace_bytes, void* stream) {
    return gemm_dx_impl(d, M, dY, Wq, sw, A, nullptr, dX, workspace, workspace_bytes, stream);
}

int qlora_gemm_dx_relu(const qlora_layer_desc* d, int M, const void* dY, const int8_t* Wq,
                       const float* sw, const float* A, const void* X, void* dX,
                       const void* workspace, size_t workspace_bytes, void* stream) {
    if (!X) return fail(QLORA_EINVAL, "NULL pointer argument");
    return gemm_dx_impl(d, M, dY, Wq, sw, A, X, dX, workspace, workspace_bytes, stream);
}

int qlora_set_rank_pass_rows(int rows) {
    if (rows < 0 || rows > (1 << 24)) return fail(QLORA_EINVAL, "rows per CTA must be in [0, 2^24]");
    return g_rank_pass_rows.exchange(rows);
}

int qlora_lora_grad_x(const qlora_layer_desc* d, int M, const void* X, float* dA,
                      const void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && dA && workspace, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(aligned(X, 16) && aligned(workspace, 256), QLORA_EALIGN,
               "X must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(dA, 4), QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) return cuda_status(cudaMemsetAsync(dA, 0, sizeof(float) * d->K * d->r, s), "memset dA");
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    int nsl = 0;
    const float* g = g_source(w, workspace, &nsl);
    return cuda_status(launch_rank_x(act_of(d), X, g, nsl, M, d->K, d->r, lora_scale(d), dA, status,
                                     s),
                       "X pass launch");
}

int qlora_forward(const qlora_layer_desc* d, int M, const void* X, const int8_t* Wq,
                  const float* sw, const float* bias, const float* A, const float* B, void* Y,
                  float* xA, void* workspace, size_t workspace_bytes, const qlora_debug* dbg,
                  void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && Wq && sw && A && B && Y && xA && workspace, QLORA_EINVAL,
               "NULL pointer argument");
    QL_REQUIRE(aligned(X, 16) && aligned(Y, 16) && aligned(Wq, 16) && aligned(workspace, 256),
               QLORA_EALIGN, "X, Y, Wq must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(sw, 4) && aligned(A, 4) && aligned(B, 4) && aligned(xA, 4) &&
                   (!bias || aligned(bias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    QL_REQUIRE(!dbg || ((!dbg->xq || aligned(dbg->xq, 16)) && (!dbg->sx || aligned(dbg->sx, 4)) &&
                        (!dbg->acc || aligned(dbg->acc, 4))),
               QLORA_EALIGN, "misaligned debug output");
    if (M == 0) return QLORA_OK;
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int8_t* Xq = (dbg && dbg->xq) ? dbg->xq : reinterpret_cast<int8_t*>(ws + w.xq);
    float* sx = (dbg && dbg->sx) ? dbg->sx : reinterpret_cast<float*>(ws + w.sx);
    rc = qlora_quantize_input(d, M, X, A, Xq, sx, xA, stream);
    if (rc != QLORA_OK) return rc;
    return qlora_gemm_forward(d, M, Xq, sx, Wq, sw, bias, xA, B, Y, dbg ? dbg->acc : nullptr,
                              stream);
}

// The backward's second stream: dX and dA both need only G and the inputs,
// so from kSideStreamMinM tokens the X pass runs on it beside the dX GEMM
// (an event fork and join, which stream capture records as two branches),
// taking the SMs the GEMM's last partial wave of tiles leaves.  One stream
// and two events per host thread and device, created on first use and kept
// for the thread's life; if they cannot be created (for instance during a
// global-mode stream capture) the backward stays on the caller's stream.
namespace {
constexpr int kSideStreamMinM = 512;
struct SideStream {
    bool tried = false;
    cudaStream_t st = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream* side_stream() {
    static thread_local SideStream per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    SideStream& ss = per_dev[dev];
    if (!ss.tried) {
        ss.tried = true;
        if (cudaStreamCreateWithFlags(&ss.st, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
            (void)cudaGetLastError();
            ss.st = nullptr;
        }
    }
    return ss.st ? &ss : nullptr;
}
}  // namespace

int qlora_backward(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                   const int8_t* Wq, const float* sw, const float* A, const float* B,
                   const float* xA, void* dX, float* dA, float* dB, float* dbias, void* workspace,
                   size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && dY && Wq && sw && A && B && xA && dA && dB && workspace, QLORA_EINVAL,
               "NULL pointer argument");
    QL_REQUIRE(aligned(X, 16) && aligned(dY, 16) && aligned(Wq, 16) && (!dX || aligned(dX, 16)) &&
                   aligned(workspace, 256),
               QLORA_EALIGN, "X, dY, dX, Wq must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(sw, 4) && aligned(A, 4) && aligned(B, 4) && aligned(xA, 4) &&
                   aligned(dA, 4) && aligned(dB, 4) && (!dbias || aligned(dbias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        // empty batch: the gradients of the LoRA factors and bias are zero
        rc = cuda_status(cudaMemsetAsync(dA, 0, sizeof(float) * d->K * d->r, s), "memset dA");
        if (rc == QLORA_OK)
            rc = cuda_status(cudaMemsetAsync(dB, 0, sizeof(float) * d->r * d->N, s), "memset dB");
        if (rc == QLORA_OK && dbias)
            rc = cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * d->N, s), "memset dbias");
        return rc;
    }
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    rc = qlora_lora_grad_dy(d, M, dY, B, xA, dB, dbias, nullptr, workspace, workspace_bytes, stream);
    if (rc != QLORA_OK) return rc;
    SideStream* ss = (dX && M >= kSideStreamMinM) ? side_stream() : nullptr;
    if (ss) {
        // G is final: the dX GEMM here (issued first, at the greatest
        // priority), the X pass on the second stream, then the join
        rc = cuda_status(cudaEventRecord(ss->fork, s), "backward fork");
        if (rc != QLORA_OK) return rc;
        rc = qlora_gemm_dx(d, M, dY, Wq, sw, A, dX, workspace, workspace_bytes, stream);
        const int rc_wait = cuda_status(cudaStreamWaitEvent(ss->st, ss->fork, 0), "backward fork");
        const int rc_x = rc_wait == QLORA_OK
                             ? qlora_lora_grad_x(d, M, X, dA, workspace, workspace_bytes, ss->st)
                             : rc_wait;
        // the join is recorded whatever happened, so the caller's stream never
        // runs ahead of work issued on the second stream
        const int rc_join = cuda_status(cudaEventRecord(ss->join, ss->st), "backward join");
        const int rc_join2 = rc_join == QLORA_OK
                                 ? cuda_status(cudaStreamWaitEvent(s, ss->join, 0), "backward join")
                                 : rc_join;
        if (rc != QLORA_OK) return rc;
        if (rc_x != QLORA_OK) return rc_x;
        return rc_join2;
    }
    if (dX) {
        rc = qlora_gemm_dx(d, M, dY, Wq, sw, A, dX, workspace, workspace_bytes, stream);
        if (rc != QLORA_OK) return rc;
    }
    return qlora_lora_grad_x(d, M, X, dA, workspace, workspace_bytes, stream);
}

int qlora_merge(const qlora_layer_desc* d, const int8_t* Wq, const float* sw, const float* A,
                const float* B, int8_t* Wq_out, float* sw_out, void* stream) {
    int rc = check_desc(d);
    if (rc != QLORA_OK) return rc;
    if (!Wq || !sw || !A || !B || !Wq_out || !sw_out)
        return fail(QLORA_EINVAL, "NULL pointer argument");
    if (!aligned(Wq, 16) || !aligned(Wq_out, 16))
        return fail(QLORA_EALIGN, "Wq and Wq_out must be 16-byte aligned");
    if (!aligned(sw, 4) || !aligned(A, 4) || !aligned(B, 4) || !aligned(sw_out, 4))
        return fail(QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    if (Wq_out == Wq || sw_out == sw) return fail(QLORA_EINVAL, "merge outputs alias its inputs");
    const float c = d->alpha / static_cast<float>(d->r);
    return cuda_status(launch_merge(Wq, sw, A, B, d->K, d->N, d->r, c, Wq_out, sw_out,
                                    static_cast<cudaStream_t>(stream)),
                       "merge launch");
}

// ---------------------------------------------------------------------------
// packed int4 kernels
// ---------------------------------------------------------------------------
static int check_int4_shape(int K, int N) {
    if (K < 1 || N < 1) return fail(QLORA_ESHAPE, "K and N must be >= 1");
    if (K % 32 != 0)
        return fail(QLORA_EUNSUPPORTED, "packed int4 kernels need K a multiple of 32 (16-byte rows of codes)");
    return QLORA_OK;
}

int qlora_quantize_weight_int4(const float* W, int K, int N, uint8_t* Wp, float* sw, void* stream) {
    if (!W || !Wp || !sw) return fail(QLORA_EINVAL, "NULL pointer argument");
    int rc = check_int4_shape(K, N);
    if (rc != QLORA_OK) return rc;
    if (!aligned(W, 4) || !aligned(sw, 4) || !aligned(Wp, 16))
        return fail(QLORA_EALIGN, "misaligned pointer (W, sw 4 B; Wp 16 B)");
    return cuda_status(launch_quantize_weight_int4(W, K, N, Wp, sw, static_cast<cudaStream_t>(stream)),
                       "quantize_weight_int4 launch");
}

int qlora_unpack_int4(const uint8_t* Wp, int K, int N, int8_t* Wq, void* stream) {
    if (!Wp || !Wq) return fail(QLORA_EINVAL, "NULL pointer argument");
    int rc = check_int4_shape(K, N);
    if (rc != QLORA_OK) return rc;
    if (!aligned(Wp, 16) || !aligned(Wq, 16)) return fail(QLORA_EALIGN, "Wp and Wq must be 16-byte aligned");
    return cuda_status(launch_unpack_int4(Wp, K, N, Wq, static_cast<cudaStream_t>(stream)),
                       "unpack_int4 launch");
}

int qlora_gemm_forward_int4(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                            const uint8_t* Wp, const float* sw, const float* bias, const float* xA,
                            const float* B, void* Y, int32_t* acc, void* stream) {
    return gemm_forward_impl(d, M, Xq, sx, reinterpret_cast<const int8_t*>(Wp), sw, bias, xA, B, Y,
                             acc, 0, stream, true);
}

int qlora_gemm_dx_int4(const qlora_layer_desc* d, int M, const void* dY, const uint8_t* Wp,
                       const float* sw, const float* A, void* dX, const void* workspace,
                       size_t workspace_bytes, void* stream) {
    return gemm_dx_impl(d, M, dY, reinterpret_cast<const int8_t*>(Wp), sw, A, nullptr, dX, workspace,
                        workspace_bytes, stream, true);
}

int qlora_merge_int4(const qlora_layer_desc* d, const uint8_t* Wp, const float* sw, const float* A,
                     const float* B, uint8_t* Wp_out, float* sw_out, void* stream) {
    int rc = check_desc(d);
    if (rc != QLORA_OK) return rc;
    rc = check_int4_shape(d->K, d->N);
    if (rc != QLORA_OK) return rc;
    if (!Wp || !sw || !A || !B || !Wp_out || !sw_out) return fail(QLORA_EINVAL, "NULL pointer argument");
    if (!aligned(Wp, 16) || !aligned(Wp_out, 16))
        return fail(QLORA_EALIGN, "Wp and Wp_out must be 16-byte aligned");
    if (!aligned(sw, 4) || !aligned(A, 4) || !aligned(B, 4) || !aligned(sw_out, 4))
        return fail(QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    if (Wp_out == Wp || sw_out == sw) return fail(QLORA_EINVAL, "merge outputs alias its inputs");
    const float c = d->alpha / static_cast<float>(d->r);
    return cuda_status(launch_merge_int4(Wp, sw, A, B, d->K, d->N, d->r, c, Wp_out, sw_out,
                                         static_cast<cudaStream_t>(stream)),
                       "merge_int4 launch");
}

// ---------------------------------------------------------------------------
// outlier-compensated int8 kernels
// ---------------------------------------------------------------------------
static long pct_index(long n, double p) {
    // the same fp64 expression as the device's percentile positions
    const double h = static_cast<double>(n - 1) * p / 100.0;
    long i = static_cast<long>(floor(h));
    return i > n - 1 ? n - 1 : i;
}

size_t qlora_outlier_cap(int K, int N) {
    if (K < 1 || N < 1) return 0;
    const long n = static_cast<long>(K) * N;
    return static_cast<size_t>((pct_index(n, 0.1) + 1) + (n - 1 - pct_index(n, 99.9)));
}

size_t qlora_outlier_workspace_bytes(int K, int N) {
    if (K < 1 || N < 1) return 0;
    return outlier_workspace_bytes(K, N);
}

static int check_outlier(const qlora_outlier_kernel* q, int K, int N) {
    QL_REQUIRE(q, QLORA_EINVAL, "NULL outlier kernel");
    QL_REQUIRE(q->codes_nk && q->codes_kn && q->par && q->start_nk && q->ent_nk && q->start_kn &&
                   q->ent_kn,
               QLORA_EINVAL, "NULL member of the outlier kernel");
    QL_REQUIRE(aligned(q->codes_nk, 16) && aligned(q->codes_kn, 16), QLORA_EALIGN,
               "outlier codes must be 16-byte aligned");
    QL_REQUIRE(aligned(q->par, 4) && aligned(q->start_nk, 4) && aligned(q->ent_nk, 4) &&
                   aligned(q->start_kn, 4) && aligned(q->ent_kn, 4),
               QLORA_EALIGN, "outlier tables must be 4-byte aligned");
    QL_REQUIRE(q->cap >= 0 && static_cast<size_t>(q->cap) >= qlora_outlier_cap(K, N), QLORA_EINVAL,
               "outlier capacity below qlora_outlier_cap(K, N)");
    return QLORA_OK;
}

int qlora_outlier_quantize(const float* W, int K, int N, const qlora_outlier_kernel* q,
                           void* workspace, size_t workspace_bytes, void* stream) {
    QL_REQUIRE(W && workspace, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(K >= 1 && N >= 1, QLORA_ESHAPE, "K and N must be >= 1");
    QL_REQUIRE(static_cast<long>(K) * N < (1L << 31), QLORA_ESHAPE, "K * N must be below 2^31");
    int rc = check_outlier(q, K, N);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(aligned(W, 4) && aligned(workspace, 256), QLORA_EALIGN,
               "W must be 4-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(workspace_bytes >= outlier_workspace_bytes(K, N), QLORA_EINVAL, "workspace too small");
    OutlierKernel k{q->codes_nk, q->codes_kn, q->par, q->start_nk, q->ent_nk, q->start_kn, q->ent_kn,
                    q->cap};
    return cuda_status(launch_quantize_outlier(W, K, N, k, workspace, static_cast<cudaStream_t>(stream)),
                       "outlier quantizer launch");
}

int qlora_outlier_forward(const qlora_layer_desc* d, int M, const void* X,
                          const qlora_outlier_kernel* q, const float* bias, const float* A,
                          const float* B, void* Y, float* xA, void* workspace,
                          size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && A && B && Y && xA && workspace, QLORA_EINVAL, "NULL pointer argument");
    rc = check_outlier(q, d->K, d->N);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(aligned(X, 16) && aligned(Y, 16) && aligned(workspace, 256), QLORA_EALIGN,
               "X and Y must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(A, 4) && aligned(B, 4) && aligned(xA, 4) && (!bias || aligned(bias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    if (M == 0) return QLORA_OK;
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    // xA from the input pass (its int8 rows go to the workspace unused: the
    // layer's activations are not quantized)
    rc = cuda_status(launch_quantize_rows(act_of(d), X, A, M, d->K, d->r,
                                          reinterpret_cast<int8_t*>(ws + w.xq),
                                          reinterpret_cast<float*>(ws + w.sx), xA, status, s),
                     "input pass launch");
    if (rc != QLORA_OK) return rc;
    // Y = X Wr + bias + c xA B on the de-quantizing GEMM: contraction over K
    // (the rows of codes_kn), output columns N, rank-r factor B^T
    DxEpilogue ep;
    ep.Gp = xA;
    ep.ncb = 1;
    ep.A = B;
    ep.a_ks = 1;
    ep.a_js = d->N;
    ep.r = d->r;
    ep.c = lora_scale(d);
    ep.dX = Y;
    ep.gate = nullptr;
    ep.bias = bias;
    ep.ol = OutlierArgs{q->par, q->start_kn, q->ent_kn, (d->N + 127) / 128};
    return cuda_status(launch_gemm_dx(act_of(d), X, reinterpret_cast<const int8_t*>(q->codes_kn),
                                      nullptr, M, d->K, d->N, ep, status, s),
                       "outlier forward GEMM launch");
}

int qlora_outlier_backward(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                           const qlora_outlier_kernel* q, const float* A, const float* B,
                           const float* xA, void* dX, float* dA, float* dB, float* dbias,
                           void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && dY && A && B && xA && dA && dB && workspace, QLORA_EINVAL,
               "NULL pointer argument");
    rc = check_outlier(q, d->K, d->N);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(aligned(X, 16) && aligned(dY, 16) && (!dX || aligned(dX, 16)) &&
                   aligned(workspace, 256),
               QLORA_EALIGN, "X, dY, dX must be 16-byte aligned, workspace 256-byte aligned");
    QL_REQUIRE(aligned(A, 4) && aligned(B, 4) && aligned(xA, 4) && aligned(dA, 4) &&
                   aligned(dB, 4) && (!dbias || aligned(dbias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        rc = cuda_status(cudaMemsetAsync(dA, 0, sizeof(float) * d->K * d->r, s), "memset dA");
        if (rc == QLORA_OK)
            rc = cuda_status(cudaMemsetAsync(dB, 0, sizeof(float) * d->r * d->N, s), "memset dB");
        if (rc == QLORA_OK && dbias)
            rc = cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * d->N, s), "memset dbias");
        return rc;
    }
    const WsLayout w = layout_for(*d, M);
    QL_REQUIRE(workspace_bytes >= w.total, QLORA_EINVAL, "workspace too small");
    rc = qlora_lora_grad_dy(d, M, dY, B, xA, dB, dbias, nullptr, workspace, workspace_bytes, stream);
    if (rc != QLORA_OK) return rc;
    if (dX) {
        int* status = status_ptr();
        QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
        DxEpilogue ep;
        ep.Gp = g_source(w, workspace, &ep.ncb);
        ep.A = A;
        ep.r = d->r;
        ep.c = lora_scale(d);
        ep.dX = dX;
        ep.gate = nullptr;
        ep.ol = OutlierArgs{q->par, q->start_nk, q->ent_nk, (d->K + 127) / 128};
        rc = cuda_status(launch_gemm_dx(act_of(d), dY, reinterpret_cast<const int8_t*>(q->codes_nk),
                                        nullptr, M, d->N, d->K, ep, status, s),
                         "outlier dX GEMM launch");
        if (rc != QLORA_OK) return rc;
    }
    return qlora_lora_grad_x(d, M, X, dA, workspace, workspace_bytes, stream);
}

int qlora_permute(const void* src, void* dst, int ndim, const int64_t* shape, const int* perm,
                  int elem_bytes, void* stream) {
    QL_REQUIRE(src && dst && shape && perm, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(ndim >= 1 && ndim <= kMaxPermAxes, QLORA_ESHAPE, "ndim must be in [1, 8]");
    QL_REQUIRE(elem_bytes == 1 || elem_bytes == 2 || elem_bytes == 4 || elem_bytes == 8, QLORA_EINVAL,
               "elem_bytes must be 1, 2, 4 or 8");
    QL_REQUIRE(aligned(src, elem_bytes) && aligned(dst, elem_bytes), QLORA_EALIGN,
               "src and dst must be aligned to the element size");
    QL_REQUIRE(src != dst, QLORA_EINVAL, "src and dst must not alias");
    long long sh[kMaxPermAxes];
    bool seen[kMaxPermAxes] = {false};
    for (int d = 0; d < ndim; ++d) {
        QL_REQUIRE(shape[d] >= 0, QLORA_ESHAPE, "negative extent");
        QL_REQUIRE(perm[d] >= 0 && perm[d] < ndim && !seen[perm[d]], QLORA_EINVAL,
                   "perm must be a permutation of 0 .. ndim-1");
        seen[perm[d]] = true;
        sh[d] = static_cast<long long>(shape[d]);
    }
    return cuda_status(launch_permute(src, dst, ndim, sh, perm, elem_bytes, static_cast<cudaStream_t>(stream)),
                       "permute launch");
}

// ---------------------------------------------------------------------------
// the float8 recipe
// ---------------------------------------------------------------------------
int qlora_fp8_quantize(const void* T, int rows, int cols, qlora_dtype dtype, qlora_fp8_format fmt,
                       const float* scale_in, float* scale_out, float* amax_history, int history_len,
                       uint8_t* q, uint8_t* qt, void* workspace, size_t workspace_bytes, void* stream) {
    QL_REQUIRE(T && scale_in && scale_out && amax_history && q && workspace, QLORA_EINVAL,
               "NULL pointer argument");
    QL_REQUIRE(rows >= 1 && cols >= 1 && history_len >= 1, QLORA_ESHAPE,
               "rows, cols and history_len must be >= 1");
    QL_REQUIRE(static_cast<long long>(rows) * cols < (1LL << 40), QLORA_ESHAPE, "tensor too large");
    QL_REQUIRE(dtype == QLORA_F32 || dtype == QLORA_BF16, QLORA_EINVAL, "unknown dtype");
    QL_REQUIRE(fmt == QLORA_FP8_E4M3 || fmt == QLORA_FP8_E5M2, QLORA_EINVAL, "unknown float8 format");
    QL_REQUIRE(scale_out != scale_in, QLORA_EINVAL, "scale_out must not alias scale_in");
    QL_REQUIRE(aligned(T, dtype == QLORA_BF16 ? 2 : 4) && aligned(scale_in, 4) && aligned(scale_out, 4) &&
                   aligned(amax_history, 4) && aligned(workspace, 4),
               QLORA_EALIGN, "misaligned pointer");
    QL_REQUIRE(workspace_bytes >= QLORA_FP8_WORKSPACE_BYTES, QLORA_EINVAL, "workspace too small");
    return cuda_status(launch_fp8_quantize(dtype == QLORA_BF16 ? kBF16 : kF32, T, rows, cols, scale_in,
                                           scale_out, amax_history, history_len,
                                           fmt == QLORA_FP8_E4M3 ? kFp8E4M3 : kFp8E5M2, q, qt, workspace,
                                           nullptr, static_cast<cudaStream_t>(stream)),
                       "float8 quantizer launch");
}

size_t qlora_fp8_colsum_workspace_bytes(int rows, int cols) {
    if (rows < 1 || cols < 1) return 0;
    return fp8_colsum_ws_bytes(rows, cols);
}

int qlora_fp8_quantize_colsum(const void* T, int rows, int cols, qlora_dtype dtype, qlora_fp8_format fmt,
                              const float* scale_in, float* scale_out, float* amax_history, int history_len,
                              uint8_t* q, uint8_t* qt, float* colsum, void* workspace, size_t workspace_bytes,
                              void* stream) {
    QL_REQUIRE(T && scale_in && scale_out && amax_history && q && colsum && workspace, QLORA_EINVAL,
               "NULL pointer argument");
    QL_REQUIRE(rows >= 1 && cols >= 1 && history_len >= 1, QLORA_ESHAPE,
               "rows, cols and history_len must be >= 1");
    QL_REQUIRE(static_cast<long long>(rows) * cols < (1LL << 40), QLORA_ESHAPE, "tensor too large");
    QL_REQUIRE(dtype == QLORA_F32 || dtype == QLORA_BF16, QLORA_EINVAL, "unknown dtype");
    QL_REQUIRE(fmt == QLORA_FP8_E4M3 || fmt == QLORA_FP8_E5M2, QLORA_EINVAL, "unknown float8 format");
    QL_REQUIRE(scale_out != scale_in, QLORA_EINVAL, "scale_out must not alias scale_in");
    QL_REQUIRE(aligned(scale_in, 4) && aligned(scale_out, 4) && aligned(amax_history, 4) && aligned(colsum, 4) &&
                   aligned(workspace, 256),
               QLORA_EALIGN, "misaligned pointer (workspace: 256 bytes)");
    QL_REQUIRE(fp8_tiled_applies(T, rows, cols, q, qt), QLORA_EUNSUPPORTED,
               "column sums need T 16-byte aligned, cols % 8 == 0, q 8-byte aligned and qt NULL or 16-byte "
               "aligned with rows % 16 == 0");
    QL_REQUIRE(workspace_bytes >= fp8_colsum_ws_bytes(rows, cols), QLORA_EINVAL, "workspace too small");
    return cuda_status(launch_fp8_quantize(dtype == QLORA_BF16 ? kBF16 : kF32, T, rows, cols, scale_in,
                                           scale_out, amax_history, history_len,
                                           fmt == QLORA_FP8_E4M3 ? kFp8E4M3 : kFp8E5M2, q, qt, workspace,
                                           colsum, static_cast<cudaStream_t>(stream)),
                       "float8 quantizer launch");
}

static int fp8_gemm_impl(const uint8_t* A, qlora_fp8_format fmt_a, const uint8_t* B, qlora_fp8_format fmt_b,
                         int M, int N, int K, const float* scale_a, const float* scale_b, const float* bias,
                         void* C, qlora_dtype c_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    QL_REQUIRE(A && B && scale_a && scale_b && C, QLORA_EINVAL, "NULL pointer argument");
    QL_REQUIRE(M >= 1 && N >= 1 && K >= 1, QLORA_ESHAPE, "M, N and K must be >= 1");
    QL_REQUIRE(K % 16 == 0, QLORA_EUNSUPPORTED, "K must be a multiple of 16 (16-byte rows of codes)");
    QL_REQUIRE((fmt_a == QLORA_FP8_E4M3 || fmt_a == QLORA_FP8_E5M2) &&
                   (fmt_b == QLORA_FP8_E4M3 || fmt_b == QLORA_FP8_E5M2),
               QLORA_EINVAL, "unknown float8 format");
    QL_REQUIRE(c_dtype == QLORA_F32 || c_dtype == QLORA_BF16, QLORA_EINVAL, "unknown dtype");
    QL_REQUIRE(aligned(A, 16) && aligned(B, 16) && aligned(C, 16), QLORA_EALIGN,
               "A, B and C must be 16-byte aligned");
    QL_REQUIRE(aligned(scale_a, 4) && aligned(scale_b, 4) && (!bias || aligned(bias, 4)), QLORA_EALIGN,
               "fp32 vectors must be 4-byte aligned");
    QL_REQUIRE(!workspace || aligned(workspace, 256), QLORA_EALIGN, "workspace must be 256-byte aligned");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    return cuda_status(launch_fp8_gemm(A, fmt_a == QLORA_FP8_E4M3 ? kFp8E4M3 : kFp8E5M2, B,
                                       fmt_b == QLORA_FP8_E4M3 ? kFp8E4M3 : kFp8E5M2, M, N, K, scale_a,
                                       scale_b, bias, C, c_dtype == QLORA_BF16 ? kBF16 : kF32, status,
                                       static_cast<cudaStream_t>(stream), workspace, workspace_bytes),
                       "float8 GEMM launch");
}

int qlora_fp8_gemm(const uint8_t* A, qlora_fp8_format fmt_a, const uint8_t* B, qlora_fp8_format fmt_b,
                   int M, int N, int K, const float* scale_a, const float* scale_b, const float* bias,
                   void* C, qlora_dtype c_dtype, void* stream) {
    return fp8_gemm_impl(A, fmt_a, B, fmt_b, M, N, K, scale_a, scale_b, bias, C, c_dtype, nullptr, 0, stream);
}

size_t qlora_fp8_gemm_workspace_bytes(int M, int N, int K) {
    if (M < 1 || N < 1 || K < 1) return 0;
    return fp8_gemm_ws_bytes(M, N, K);
}

int qlora_fp8_gemm_ws(const uint8_t* A, qlora_fp8_format fmt_a, const uint8_t* B, qlora_fp8_format fmt_b,
                      int M, int N, int K, const float* scale_a, const float* scale_b, const float* bias,
                      void* C, qlora_dtype c_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    return fp8_gemm_impl(A, fmt_a, B, fmt_b, M, N, K, scale_a, scale_b, bias, C, c_dtype, workspace,
                         workspace_bytes, stream);
}

int qlora_selftest_wait_timeout(unsigned int limit_us, void* stream) {
    QL_REQUIRE(limit_us >= 1 && limit_us <= 2000000, QLORA_EINVAL, "limit_us must be in [1, 2e6]");
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    return cuda_status(launch_selftest_wait(status, 1000ull * limit_us,
                                            static_cast<cudaStream_t>(stream)),
                       "self-test launch");
}

int qlora_relu(void* Y, size_t n, qlora_dtype dtype, void* stream) {
    if (!Y) return fail(QLORA_EINVAL, "NULL pointer argument");
    if (dtype != QLORA_F32 && dtype != QLORA_BF16) return fail(QLORA_EINVAL, "unknown dtype");
    if (n == 0) return QLORA_OK;
    return cuda_status(launch_relu(dtype == QLORA_BF16 ? kBF16 : kF32, Y, n,
                                   static_cast<cudaStream_t>(stream)),
                       "relu launch");
}

int qlora_relu_backward(void* dY, const void* Y, size_t n, qlora_dtype dtype, void* stream) {
    if (!dY || !Y) return fail(QLORA_EINVAL, "NULL pointer argument");
    if (dtype != QLORA_F32 && dtype != QLORA_BF16) return fail(QLORA_EINVAL, "unknown dtype");
    if (n == 0) return QLORA_OK;
    return cuda_status(launch_relu_backward(dtype == QLORA_BF16 ? kBF16 : kF32, dY, Y, n,
                                            static_cast<cudaStream_t>(stream)),
                       "relu backward launch");
}

int qlora_backward_noalloc(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                           const int8_t* Wq, const float* sw, const float* A, const float* B,
                           const float* xA, void* dX, float* dA, float* dB, float* dbias,
                           void* stream) {
    int rc = check_layer(d, M);
    if (rc != QLORA_OK) return rc;
    QL_REQUIRE(X && dY && Wq && sw && A && B && xA && dA && dB, QLORA_EINVAL,
               "NULL pointer argument");
    QL_REQUIRE(aligned(X, 16) && aligned(dY, 16) && aligned(Wq, 16) && (!dX || aligned(dX, 16)),
               QLORA_EALIGN, "X, dY, dX, Wq must be 16-byte aligned");
    QL_REQUIRE(aligned(sw, 4) && aligned(A, 4) && aligned(B, 4) && aligned(xA, 4) &&
                   aligned(dA, 4) && aligned(dB, 4) && (!dbias || aligned(dbias, 4)),
               QLORA_EALIGN, "fp32 vectors must be 4-byte aligned");
    const WsLayout w = layout_for(*d, M);
    if (w.bwd_total > QLORA_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "qlora_backward_noalloc: M=%d, N=%d, r=%d needs %zu bytes of scratch, above the "
                 "%d-byte static scratch; use qlora_backward with a caller-supplied workspace",
                 M, d->N, d->r, w.bwd_total, QLORA_NOALLOC_SCRATCH_BYTES);
        return fail(QLORA_ESHAPE, msg);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {
        rc = cuda_status(cudaMemsetAsync(dA, 0, sizeof(float) * d->K * d->r, s), "memset dA");
        if (rc == QLORA_OK)
            rc = cuda_status(cudaMemsetAsync(dB, 0, sizeof(float) * d->r * d->N, s), "memset dB");
        if (rc == QLORA_OK && dbias)
            rc = cuda_status(cudaMemsetAsync(dbias, 0, sizeof(float) * d->N, s), "memset dbias");
        return rc;
    }
    uint8_t* scratch = nullptr;
    rc = cuda_status(noalloc_scratch(&scratch), "static scratch address");
    if (rc != QLORA_OK) return rc;
    int* status = status_ptr();
    QL_REQUIRE(status, QLORA_ECUDA, "no CUDA device");
    float* gp = reinterpret_cast<float*>(scratch + w.gp);
    const float c = lora_scale(d);
    rc = cuda_status(launch_rank_dy(act_of(d), dY, B, xA, M, d->N, d->r, c, gp, dB, dbias, status,
                                    s),
                     "dY pass launch");
    if (rc == QLORA_OK && w.reduce)
        rc = cuda_status(launch_g_reduce(gp, w.ncb, M, d->r, reinterpret_cast<float*>(scratch + w.g),
                                         s),
                         "G reduction launch");
    if (rc != QLORA_OK) return rc;
    int nsl = 0;
    const float* g = g_source(w, scratch, &nsl);
    if (dX) {
        DxEpilogue ep;
        ep.Gp = g;
        ep.ncb = nsl;
        ep.A = A;
        ep.r = d->r;
        ep.c = c;
        ep.dX = dX;
        ep.gate = nullptr;
        rc = cuda_status(launch_gemm_dx(act_of(d), dY, Wq, sw, M, d->N, d->K, ep, status, s),
                         "dX GEMM launch");
        if (rc != QLORA_OK) return rc;
    }
    return cuda_status(launch_rank_x(act_of(d), X, g, nsl, M, d->K, d->r, c, dA, status, s),
                       "X pass launch");
}

}  // extern "C"
