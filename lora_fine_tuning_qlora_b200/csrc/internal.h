// internal.h -- launchers shared between the kernel files and the C ABI
// (qlora_api.cu).  Nothing here is exported from libqlora.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qlora {

enum Act { kF32 = 0, kBF16 = 1 };

// ---------------------------------------------------------------- K1 / a0
// Xq, sx (bit-exact quantization) and xA = X . A, one pass over X.
cudaError_t launch_quantize_rows(Act act, const void* X, const float* A, int M, int K, int r,
                                 int8_t* Xq, float* sx, float* xA, int* status, cudaStream_t s);
// W [K,N] fp32 -> Wq [N,K], sw [N].
cudaError_t launch_quantize_weight(const float* W, int K, int N, int8_t* Wq, float* sw,
                                   cudaStream_t s);

// ---------------------------------------------------------------- K2
struct FwdEpilogue {
    const float* sx;    // [M]
    const float* sw;    // [N]
    const float* bias;  // [N] or null
    const float* xA;    // [M,r]
    const float* B;     // [r,N]
    int r;
    float c;
    void* Y;            // [M,N] act
    int32_t* acc;       // [M,N] debug copy or null
    int relu;           // 1: Y = max(Y, 0) (the ReLU that follows the layer in an MLP)
};
// Y = (Xq Wq^T) sx sw + bias + c xA B with the tcgen05 int8 GEMM.
// w4: Wq holds packed int4 codes [N, K/2] (K % 32 == 0), expanded in shared memory.
cudaError_t launch_gemm_i8_fwd(Act act, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                               const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4 = false);

// The forward GEMM on CTA pairs (256 x 256 tiles, k2_gemm_i8_pair.cu): bf16
// outputs, rank <= 16, at least one wave of pair tiles.
bool gemm_fwd_pair_applies(Act act, int M, int N, int K, int r);
cudaError_t launch_gemm_i8_fwd_pair(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                    const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4);

// ---------------------------------------------------------------- K3
// Outlier-compensated int8 kernel as a GEMM operand (outlier.cu): uint8
// affine codes [rows, cols] with rows the contraction, one scale and bias per
// tensor (par[2], par[3]), and the fp16 outliers of every (row, 128-column
// block) in ent[start[row * nb + block] .. start[row * nb + block + 1]), each
// (column within the block << 16) | fp16 bits.
struct OutlierArgs {
    const float* par;
    const int* start;
    const uint32_t* ent;
    int nb;  // 128-column blocks per row
};

struct DxEpilogue {
    const float* Gp;  // [ncb][M,r] slices of G = dY B^T (G = sum of the slices)
    int ncb;
    const float* A;   // element (k, j) at A[k * a_ks + j * a_js]; [K,r] when a_ks = 0
    int r;
    float c;
    void* dX;         // [M,K] act
    const void* gate; // [M,K] act or null: dX = 0 where gate <= 0 (the layer input came
                      // out of a ReLU, whose backward this applies)
    int a_ks = 0;     // 0: r
    int a_js = 1;
    const float* bias = nullptr;      // [K] added per output column, or null
    OutlierArgs ol{};  // ol.par != nullptr: outlier-compensated codes instead of int8 / int4
};

// The one-off quantization of an outlier-compensated int8 kernel W [K,N]
// (outlier.cu): codes in both layouts, affine parameters, bucketed outliers.
struct OutlierKernel {
    uint8_t* codes_nk;  // [N,K]
    uint8_t* codes_kn;  // [K,N]
    float* par;         // [4] lo, hi, scale, bias
    int* start_nk;      // [N * ceil(K/128) + 1]
    uint32_t* ent_nk;   // [cap]
    int* start_kn;      // [K * ceil(N/128) + 1]
    uint32_t* ent_kn;   // [cap]
    int cap;
};
size_t outlier_buckets_nk(int K, int N);
size_t outlier_buckets_kn(int K, int N);
size_t outlier_workspace_bytes(int K, int N);
cudaError_t launch_quantize_outlier(const float* W, int K, int N, const OutlierKernel& q,
                                    void* workspace, cudaStream_t s);
// dX = dY (Wq sw)^T + c G A^T.  tcgen05 bf16 path when possible, else SIMT.
// w4: Wq holds packed int4 codes [N, K/2] (K % 32 == 0).
cudaError_t launch_gemm_dx(Act act, const void* dY, const int8_t* Wq, const float* sw, int M,
                           int N, int K, const DxEpilogue& ep, int* status, cudaStream_t s,
                           bool w4 = false);
// The bf16 dX GEMM on CTA pairs (256 x 256 tiles, k3_dx_pair.cu): for N a
// multiple of 64, rank <= 16 and at least one wave of pair tiles.
bool gemm_dx_pair_applies(int M, int N, int K, int r);
cudaError_t launch_gemm_dx_pair(const void* dY, const int8_t* Wq, const float* sw, int M, int N,
                                int K, const DxEpilogue& ep, int* status, cudaStream_t s, bool w4);

// Few tokens (M <= 64, rank <= 16, fewer large tiles than SMs): tokens on
// the MMA's N, output channels on its M, the contraction split over a
// cluster (small_m.cu).  int8 or packed int4 codes (w4) with a scale per
// row; not the outlier-compensated kernels.
bool small_m_applies(int M, int out_channels, int r);
cudaError_t launch_gemm_i8_fwd_small(Act act, const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                     const FwdEpilogue& ep, int* status, cudaStream_t s, bool w4);
cudaError_t launch_gemm_dx_small(const void* dY, const int8_t* Wq, const float* sw, int M, int N, int K,
                                 const DxEpilogue& ep, int* status, cudaStream_t s, bool w4);

// Axis permutation of a row-major tensor of up to kMaxPermAxes axes
// (permute.cu): dst axis d is src axis perm[d].
constexpr int kMaxPermAxes = 8;
cudaError_t launch_permute(const void* src, void* dst, int nd, const long long* shape, const int* perm,
                           int elem_bytes, cudaStream_t s);

// The float8 recipe (fp8.cu).  Formats of the codes:
constexpr int kFp8E4M3 = 0;
constexpr int kFp8E5M2 = 1;
// Codes of T [R, Cc] with the stored scale *scale_in (row-major q and, if
// qt != null, transposed qt [Cc, R]); then *scale_out and the history hist
// [L] of delayed scaling.  ws: device scratch (the amax word; with column
// sums, fp8_colsum_ws_bytes).  colsum [Cc] (optional): the column sums of T
// in fp32.
cudaError_t launch_fp8_quantize(Act act, const void* T, int R, int Cc, const float* scale_in, float* scale_out,
                                float* hist, int L, int fmt, uint8_t* q, uint8_t* qt, void* ws, float* colsum,
                                cudaStream_t s);
// Whether the 128 x 128 tiled quantizer takes this layout (T 16-byte
// aligned, Cc % 8 == 0, q 8-byte aligned, qt null or 16-byte aligned with
// R % 16 == 0); column sums need it.
bool fp8_tiled_applies(const void* T, int R, int Cc, const uint8_t* q, const uint8_t* qt);
// Workspace bytes of a quantization with column sums of T [R, Cc].
size_t fp8_colsum_ws_bytes(int R, int Cc);
// C [M,N] = (A [M,K] B [N,K]^T) * sa * sb (+ bias [N]); K-major fp8 codes.
cudaError_t launch_fp8_gemm(const uint8_t* A, int afmt, const uint8_t* B, int bfmt, int M, int N, int K,
                            const float* sa, const float* sb, const float* bias, void* C, Act out, int* status,
                            cudaStream_t s, void* ws = nullptr, size_t ws_bytes = 0);
// Workspace bytes that let launch_fp8_gemm split the CTA pairs' partial last
// wave of tiles (0: no split at this shape on this device).
size_t fp8_gemm_ws_bytes(int M, int N, int K);

// ---------------------------------------------------------------- K4
// The dY pass runs on the tensor cores for bf16 activations whose rows TMA
// can describe (N a multiple of 8), in 128-column blocks; otherwise on CUDA
// cores in 64-column blocks.  The X pass likewise (K is always a multiple of 16).
bool rank_dy_tc(Act act, int N);
// Column blocks of the dY pass = number of G slices it writes.
int rank_col_blocks(Act act, int N);
// Consumers add up to this many G slices themselves; above it the slices are
// added once into G (launch_g_reduce) and the consumers read G.
constexpr int kMaxDirectSlices = 8;

// Pass over dY: G slices into Gp, final dB and dbias.  Gp or dB may be null
// (that half is skipped); dbias may be null.
cudaError_t launch_rank_dy(Act act, const void* dY, const float* B, const float* xA, int M, int N,
                           int r, float c, float* Gp, float* dB, float* dbias, int* status,
                           cudaStream_t s);
// G [M,r] = the ncb slices of Gp added in ascending order.
cudaError_t launch_g_reduce(const float* Gp, int ncb, int M, int r, float* G, cudaStream_t s);
// Pass over X: final dA from X and G given as nsl slices (nsl = 1: G itself).
cudaError_t launch_rank_x(Act act, const void* X, const float* G, int nsl, int M, int K, int r,
                          float c, float* dA, int* status, cudaStream_t s);

// tensor-core passes (k4_rank_tc.cu)
int rank_tc_col_blocks(int C);
cudaError_t launch_rank_dy_tc(const void* dY, const float* B, const float* xA, int M, int N, int r,
                              float c, float* Gp, float* dB, float* dbias, int* status,
                              cudaStream_t s);
cudaError_t launch_rank_x_tc(const void* X, const float* G, int nsl, int M, int K, int r, float c,
                             float* dA, int* status, cudaStream_t s);

// ---------------------------------------------------------------- KM
cudaError_t launch_merge_int4(const uint8_t* Wp, const float* sw, const float* A, const float* B,
                              int K, int N, int r, float c, uint8_t* Wp_out, float* sw_out,
                              cudaStream_t s);
// Packed int4 kernels (two codes per byte, even k in the low nibble; K % 32 == 0).
cudaError_t launch_quantize_weight_int4(const float* W, int K, int N, uint8_t* Wp, float* sw,
                                        cudaStream_t s);
cudaError_t launch_unpack_int4(const uint8_t* Wp, int K, int N, int8_t* Wq, cudaStream_t s);
cudaError_t launch_merge(const int8_t* Wq, const float* sw, const float* A, const float* B, int K,
                         int N, int r, float c, int8_t* Wq_out, float* sw_out, cudaStream_t s);

// ---------------------------------------------------------------- ReLU
cudaError_t launch_relu(Act act, void* y, size_t n, cudaStream_t s);
cudaError_t launch_relu_backward(Act act, void* g, const void* h, size_t n, cudaStream_t s);

// ---------------------------------------------------------------- self test
// A kernel whose bounded wait runs out after limit_ns (records a timeout).
cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t s);

// ---------------------------------------------------------------- TMA maps
// Encodes a 2D row-major tensor map: `rows` x `cols` elements of `elem`
// bytes, row pitch `pitch_bytes`, box `box_rows` x `box_cols`.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t rows, uint64_t cols, uint64_t pitch_bytes, uint32_t box_rows,
                  uint32_t box_cols, CUtensorMapSwizzle swizzle);
// A [rows, cols] row-major matrix seen as [rows][cols / blk][blk] (cols a
// multiple of blk), 128-byte swizzle: one box of box_blocks consecutive
// blk-wide column blocks x box_rows rows lands as box_blocks [box_rows x blk]
// tiles one after another in shared memory.
bool make_tmap_3d_blocks(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, uint64_t rows, uint64_t cols, uint32_t blk,
                         uint32_t box_rows, uint32_t box_blocks);

// Number of SMs of the current device (cached per device).
int sm_count();

// Launches `kern` with programmatic stream serialization (the kernel starts
// while its predecessor drains; it calls pdl_wait() before touching global
// memory), optionally as thread-block clusters of cluster_y CTAs along y.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     int cluster_y, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_y > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = cluster_y;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Minimum rows per CTA of the column-sum passes (dB/dbias, dA); 0 = default.
int rank_pass_rows();

// launch_k with thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_kx(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The device's greatest (most urgent) stream priority, looked up once.
int greatest_priority();

// launch_kx at the device's greatest priority: when kernels of several
// streams are ready at once, this one's CTAs are placed first.
template <typename... KArgs, typename... Args>
cudaError_t launch_kx_urgent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[3];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    attr[2].id = cudaLaunchAttributePriority;
    attr[2].val.priority = greatest_priority();
    cfg.attrs = attr;
    cfg.numAttrs = 3;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Sets the dynamic shared memory limit of `func` once per device.
cudaError_t ensure_smem_attr(const void* func, int bytes);

}  // namespace qlora
