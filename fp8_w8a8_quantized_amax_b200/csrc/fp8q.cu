// fp8q.cu -- C ABI of libfp8q.so: argument checks, tensor maps, dispatch.
//
// All device work lives in the kernels included below; this file only checks
// arguments (before anything touches CUDA), builds TMA descriptors, picks a
// kernel and launch shape, and maps errors to fp8q_status.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/fp8q.h"
#include "calib.cuh"
#include "gemm_decode.cuh"
#include "gemm_prefill.cuh"
#include "gemv_w8a16.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

using fp8q::decode::Params;

constexpr int kMaxDevices = 64;
constexpr int64_t kInt32Max = 2147483647;

fp8q_status noalloc_reset_current_device();

// ------------------------------------------------------------ device info ---

struct DeviceInfo {
  int sms = 0;
  bool ready = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

fp8q_status current_device(int* dev, int* sms) {
  if (cudaGetDevice(dev) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FP8Q_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[*dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) return FP8Q_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess) return FP8Q_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess) return FP8Q_ERR_CUDA;
    if (major != 10 || minor != 0) return FP8Q_ERR_UNSUPPORTED;   // built for sm_100a only
    d.ready = true;
  }
  *sms = d.sms;
  return FP8Q_OK;
}

// Opt a kernel in to large dynamic shared memory, once per (kernel, device).
struct SmemOptIn {
  const void* fn;
  int dev;
};
SmemOptIn g_optin[256];
int g_noptin = 0;
std::mutex g_optin_mu;

template <typename K>
fp8q_status ensure_smem(K kernel, int bytes, int dev) {
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lk(g_optin_mu);
  for (int i = 0; i < g_noptin; ++i)
    if (g_optin[i].fn == fn && g_optin[i].dev == dev) return FP8Q_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (g_noptin < 256) g_optin[g_noptin++] = {fn, dev};
  return FP8Q_OK;
}

// cluster_x > 0: launched in clusters of cluster_x CTAs (for kernels without
// a compile-time cluster shape).
template <typename... KArgs, typename... Args>
fp8q_status launch_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, void* stream,
                             int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  // Programmatic dependent launch: the kernel may begin while its stream
  // predecessor finishes; every kernel here waits (griddepcontrol.wait)
  // before touching global memory.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster_x > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

template <typename... KArgs, typename... Args>
fp8q_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, void* stream, Args... args) {
  return launch_clustered(kernel, grid, block, smem, stream, 0, args...);
}

// ------------------------------------------------------------ tensor maps ---

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

fp8q_status get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Row-major uint8 matrix [rows, cols] with row stride `ld` bytes, tiles of
// box_rows x 128 bytes, 128-byte swizzle (the layout tcgen05 descriptors expect).
fp8q_status tmap_u8_sw128(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                          uint32_t box_rows) {
  if (get_encode() != FP8Q_OK) return FP8Q_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Row-major bf16 matrix [rows, cols], row stride `ld` elements, tiles of
// box_rows x 32 columns (64 bytes) with the 64-byte swizzle.
fp8q_status tmap_bf16_sw64(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                           uint32_t box_rows) {
  if (get_encode() != FP8Q_OK) return FP8Q_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {32u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Row-major bf16 matrix [rows, cols], row stride `ld` elements, tiles of
// box_rows x 64 values (128 bytes) with the 128-byte swizzle: a tcgen05 operand.
fp8q_status tmap_bf16_sw128(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                            uint32_t box_rows) {
  if (get_encode() != FP8Q_OK) return FP8Q_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ------------------------------------------------------------ quantization ---

// A mode is FP8Q_CHANNEL_TOKEN or FP8Q_BLOCK128, optionally OR'ed with FP8Q_SCALE_BF16.
bool valid_mode(int mode) {
  const int base = mode & ~FP8Q_SCALE_BF16;
  return base == FP8Q_CHANNEL_TOKEN || base == FP8Q_BLOCK128;
}

fp8q_status check_quant_args(const void* src, int64_t rows, int64_t K, int64_t ld, int mode, const uint8_t* q,
                             int64_t ldq, const float* s) {
  if (!valid_mode(mode)) return FP8Q_ERR_INVALID_ARG;
  mode &= ~FP8Q_SCALE_BF16;
  if (rows < 0 || K <= 0 || ld < K || ldq < K) return FP8Q_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (mode == FP8Q_BLOCK128 && K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (rows == 0) return FP8Q_OK;
  if (!src || !q || !s) return FP8Q_ERR_INVALID_ARG;
  if (ld % 8 != 0 || ldq % 16 != 0) return FP8Q_ERR_MISALIGNED;
  if (!aligned(src, 16) || !aligned(q, 16) || !aligned(s, 4)) return FP8Q_ERR_MISALIGNED;
  if (rows > kInt32Max || K > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  return FP8Q_OK;
}

fp8q_status launch_rows(const uint16_t* x, int64_t rows, int K, int64_t ldx, uint8_t* q, int64_t ldq, float* s,
                        bool s16, void* stream) {
  const int nvec = K / 8;
  int T = 32 * ((nvec + 32 * 8 - 1) / (32 * 8));
  if (T > 1024) T = 1024;
  const int need = (nvec + T - 1) / T;
  const dim3 grid(static_cast<unsigned>(rows));
  const dim3 block(T);
  if (need <= 1) return launch(fp8q::quant_rows_kernel<1>, grid, block, 0, stream, x, K, ldx, q, ldq, s, s16);
  if (need <= 2) return launch(fp8q::quant_rows_kernel<2>, grid, block, 0, stream, x, K, ldx, q, ldq, s, s16);
  if (need <= 4) return launch(fp8q::quant_rows_kernel<4>, grid, block, 0, stream, x, K, ldx, q, ldq, s, s16);
  if (need <= 8) return launch(fp8q::quant_rows_kernel<8>, grid, block, 0, stream, x, K, ldx, q, ldq, s, s16);
  if (need <= 16) return launch(fp8q::quant_rows_kernel<16>, grid, block, 0, stream, x, K, ldx, q, ldq, s, s16);
  return FP8Q_ERR_UNSUPPORTED;   // K > 131072
}

fp8q_status launch_rmsnorm_rows(const uint16_t* x, const uint16_t* gamma, int64_t rows, int K, int64_t ldx,
                                float eps, uint8_t* q, int64_t ldq, float* s, float* rstd, void* stream) {
  const int nvec = K / 8;
  int T = 32 * ((nvec + 32 * 8 - 1) / (32 * 8));
  if (T > 512) T = 512;
  const int need = (nvec + T - 1) / T;
  const dim3 grid(static_cast<unsigned>(rows));
  const dim3 block(T);
#define FP8Q_RMS(V)                                                                                             \
  return launch(fp8q::rmsnorm_quant_rows_kernel<V>, grid, block, 0, stream, x, gamma, K, ldx, eps, q, ldq, s, \
                rstd)
  if (need <= 1) FP8Q_RMS(1);
  if (need <= 2) FP8Q_RMS(2);
  if (need <= 4) FP8Q_RMS(4);
  if (need <= 8) FP8Q_RMS(8);
  if (need <= 16) FP8Q_RMS(16);
#undef FP8Q_RMS
  return FP8Q_ERR_UNSUPPORTED;   // K > 65536
}

// ------------------------------------------------------------------ linear ---

constexpr int kPrefillBN = 256;
constexpr int kPairStages = 6;

// Prefill kernel choice (both modes): the CTA-pair kernel for M >= 256,
// else the single-CTA kernel.  FP8Q_PREFILL_KERNEL=single|pair forces one
// (read once), for comparing them on the same problem.
int prefill_choice() {
  static int choice = [] {
    const char* e = getenv("FP8Q_PREFILL_KERNEL");
    if (e && strcmp(e, "single") == 0) return 1;
    if (e && strcmp(e, "pair") == 0) return 2;
    return 0;
  }();
  return choice;
}

constexpr int kPrefillStages = 4;
constexpr int kBlockStages = 6;
template <int NX>
constexpr int decode_stages() { return NX == 16 ? 12 : (NX == 32 ? 10 : 8); }
constexpr int kDecodeMaxM = 64;

int decode_nx(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

bool decode_half_stages(int nx);

// Stream-K split of a small-M problem: n_tiles weight tiles of 128 rows, KB K
// blocks each, over G CTAs, one per SM.  Where the kernel is built for two
// CTAs per SM (`two_per_sm`), G = c * n_tiles instead for the smallest c >= 2
// that divides KB and gives more CTAs than SMs but at most two per SM: every
// CTA streams exactly 1/c of one tile.  Measured on the Llama-3.1-70B decode
// shapes against one CTA per SM (ranges that cross tiles): qkv_proj (80
// tiles, c = 2: 160 CTAs of 32 K blocks) 0.59 -> 0.62 of HBM at M = 1, 0.58
// -> 0.61 at M = 8; down_proj (64 tiles of 224 K blocks, c = 4: 256 CTAs of
// 56) 0.74 -> 0.77 at M = 1, 0.74 -> 0.76 at M = 8; gate/up (224 tiles) take
// no c.
void decode_shape(int64_t M, int64_t N, int64_t K, int sms, bool two_per_sm, int* n_tiles, int64_t* total, int* G,
                  int* nx) {
  const int KB = static_cast<int>((K + 127) / 128);
  *n_tiles = static_cast<int>((N + 127) / 128);
  *total = static_cast<int64_t>(*n_tiles) * KB;
  *G = static_cast<int>(*total < sms ? *total : sms);
  *nx = decode_nx(M);
  if (two_per_sm)
    for (int c = 2; c * *n_tiles <= 2 * sms; ++c)
      if (c * *n_tiles > sms && KB % c == 0) {
        *G = c * *n_tiles;
        break;
      }
}

// Decode workspace: [n_tiles][4] arrival counters, padded to 16 bytes, then
// [(n_tiles + G - 1)][nx][128] fp32 partial sums.  All zero between calls.
size_t decode_counter_bytes(int n_tiles) { return (static_cast<size_t>(n_tiles) * 4 * sizeof(unsigned) + 15) & ~size_t(15); }

size_t decode_workspace_bytes(int n_tiles, int G, int nx) {
  return decode_counter_bytes(n_tiles) + static_cast<size_t>(n_tiles + G - 1) * nx * 128 * sizeof(float);
}

void decode_bind_workspace(Params& p, void* ws, void* Y, int64_t ldy) {
  p.count = static_cast<unsigned*>(ws);
  p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + decode_counter_bytes(p.n_tiles));
  p.y = static_cast<__nv_bfloat16*>(Y);
  p.ldy = ldy;
}

fp8q_status check_linear_args(const uint8_t* Xq, const float* xs, const uint8_t* Wq, const float* ws, int64_t M,
                              int64_t N, int64_t K, int mode, const void* Y, int64_t ldy) {
  if (!valid_mode(mode)) return FP8Q_ERR_INVALID_ARG;
  mode &= ~FP8Q_SCALE_BF16;
  if (M < 0 || N <= 0 || K <= 0 || ldy < N) return FP8Q_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (mode == FP8Q_BLOCK128 && K % 128 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!Xq || !xs || !Wq || !ws || !Y) return FP8Q_ERR_INVALID_ARG;
  if (ldy % 8 != 0) return FP8Q_ERR_MISALIGNED;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(xs, 4) || !aligned(ws, 4))
    return FP8Q_ERR_MISALIGNED;
  if (M > kInt32Max || N > kInt32Max || K > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  return FP8Q_OK;
}

// In-kernel sums: a warp that finds every other part of its tile already in
// loads them while its own MMAs finish (gemm_decode.cuh).  Measured on the
// 70B decode shapes on one box (back to back), it pays where every CTA streams
// at least a tile's worth of K blocks (gate/up: 0.76 -> 0.78 of HBM) and costs
// where the ranges are shorter than a tile (qkv 0.59 -> 0.58, down 0.74 ->
// 0.735): there the counter read sits in front of most segments' drains.
// FP8Q_DECODE_EARLY=0|1 forces it off or on (read once).
int decode_early_forced() {
  static int v = [] {
    const char* e = getenv("FP8Q_DECODE_EARLY");
    if (e && strcmp(e, "0") == 0) return 0;
    if (e && strcmp(e, "1") == 0) return 1;
    return -1;
  }();
  return v;
}
bool decode_early(int64_t total, int G, int KB) {
  const int f = decode_early_forced();
  return f >= 0 ? f == 1 : total / G >= KB;
}

// Where the decode kernel's split weight tiles are summed (gemm_decode.cuh).
// Measured on the Llama-3.1-70B and -3.2-3B decode shapes: in channel mode
// with up to 16 tokens the in-kernel sums (last arriver) are cheap enough to
// win everywhere; with 32 or 64 tokens only when every CTA streams at least a
// tile's worth of steps after them.  In block mode the last arriver's fence,
// atomic and loads sit at the end of a short kernel, and the reduction kernel
// pays a grid boundary; cluster split-K (one weight tile per cluster, sums in
// distributed shared memory) avoids both wherever its clusters fill most
// SMs at once.  FP8Q_DECODE_SUMS=separate|kernel|cluster forces one (read
// once; cluster where some cluster size fits, else the default), for
// comparing them on the same problem.
int decode_sums_forced() {
  static int choice = [] {
    const char* e = getenv("FP8Q_DECODE_SUMS");
    if (e && strcmp(e, "separate") == 0) return fp8q::decode::kSumsSeparate;
    if (e && strcmp(e, "kernel") == 0) return fp8q::decode::kSumsKernel;
    if (e && strcmp(e, "cluster") == 0) return fp8q::decode::kSumsCluster;
    return -1;
  }();
  return choice;
}

// Clusters of C decode CTAs (one CTA per SM) that fit on the device at once,
// per token tile, cluster size and device; 0 where the query fails.
template <int NX>
int decode_max_clusters(int C, int dev, int sms) {
  constexpr int kDecodeStages = decode_stages<NX>();
  using L = fp8q::decode::Layout<NX, kDecodeStages>;
  static std::atomic<int> cache[9][kMaxDevices];   // value + 1; 0 = not asked yet
  int v = cache[C][dev].load(std::memory_order_relaxed);
  if (v == 0) {
    auto k = fp8q::decode::gemm_decode_kernel<NX, kDecodeStages, true, fp8q::decode::kSumsCluster>;
    int n = 0;
    if (ensure_smem(k, L::kBytes, dev) == FP8Q_OK) {
      cudaLaunchConfig_t qc = {};
      qc.gridDim = dim3(static_cast<unsigned>(C * sms));
      qc.blockDim = dim3(L::kThreads);
      qc.dynamicSmemBytes = L::kBytes;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = static_cast<unsigned>(C);
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      qc.attrs = a;
      qc.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, k, &qc) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
    }
    v = n + 1;
    cache[C][dev].store(v, std::memory_order_relaxed);
  }
  return v - 1;
}

// Cluster size for cluster split-K, or 0: C in [2, 8], at most KB (every CTA
// gets a K block) and at most sms / n_tiles, the largest whose n_tiles
// clusters the device holds at once (asked of the one-CTA-per-SM build, so
// that every CTA of a cluster gets an SM of its own); by default only where
// those n_tiles * C CTAs fill at least 3/4 of the SMs.  Clusters twice as
// large, planned for two CTAs per SM, measured slower on the 3B FP8-Block
// decode shapes (0.38 -> 0.35 of HBM).
template <int NX>
int decode_cluster_size(const Params& p, int sms, int dev, bool forced) {
  int C = sms / p.n_tiles;
  if (C > 8) C = 8;
  if (C > p.KB) C = p.KB;
  for (; C >= 2; --C) {
    if (!forced && 4 * p.n_tiles * C < 3 * sms) return 0;
    if (decode_max_clusters<NX>(C, dev, sms) >= p.n_tiles) return C;
  }
  return 0;
}

// Half the stages (and at most two CTAs' worth of registers, so the early
// loads of the last contributor's partners are left out) let two decode CTAs
// share an SM: the next kernel's CTAs start beside this kernel's last ones
// (programmatic dependent launch), so their set-up and first loads overlap
// its tail.  Measured on the Llama-3.1-70B decode shapes back to back, with
// 16-token tiles: qkv 0.567 -> 0.594 of HBM at M=1, down 0.73 -> 0.75,
// gate/up unchanged, the 3B FP8-Block M=1/16 0.37 -> 0.38; with 64-token
// tiles (4 stages, and two CTAs no longer fit in tensor memory) slower: down
// 0.67 -> 0.50, qkv 0.46 -> 0.35.  So by default 16-token tiles only.
// FP8Q_DECODE_STAGES=full|half (read once) forces one form for every tile.
bool decode_half_stages(int nx) {
  static int choice = [] {
    const char* e = getenv("FP8Q_DECODE_STAGES");
    if (e && strcmp(e, "full") == 0) return 1;
    if (e && strcmp(e, "half") == 0) return 2;
    return 0;
  }();
  return choice == 2 || (choice == 0 && nx == 16);
}

template <int NX, int kDecodeStages, int MINB>
fp8q_status launch_decode_nx_s(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int mode, int dev,
                               int sms, void* stream);

template <int NX>
fp8q_status launch_decode_nx(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int mode, int dev,
                             int sms, void* stream) {
  if (decode_half_stages(NX))
    return launch_decode_nx_s<NX, decode_stages<NX>() / 2, 2>(tw, tx, p, mode, dev, sms, stream);
  return launch_decode_nx_s<NX, decode_stages<NX>(), 1>(tw, tx, p, mode, dev, sms, stream);
}

template <int NX, int kDecodeStages, int MINB>
fp8q_status launch_decode_nx_s(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int mode, int dev,
                               int sms, void* stream) {
  using namespace fp8q::decode;
  using L = Layout<NX, kDecodeStages>;
  fp8q_status st;
  const bool block = mode == FP8Q_BLOCK128;
  const int forced = decode_sums_forced();
  if (forced == kSumsCluster || (forced < 0 && block)) {
    const int C = decode_cluster_size<NX>(p, sms, dev, forced == kSumsCluster);
    if (C >= 2) {
      auto k = block ? gemm_decode_kernel<NX, kDecodeStages, true, kSumsCluster, 0, MINB>
                     : gemm_decode_kernel<NX, kDecodeStages, false, kSumsCluster, 0, MINB>;
      if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
      Params q = p;
      q.G = p.n_tiles * C;
      return launch_clustered(k, dim3(q.G), dim3(L::kThreads), L::kBytes, stream, C, tw, tx, q);
    }
  }
  const bool in_kernel = forced == kSumsKernel ||
                         (forced != kSumsSeparate && !block && (NX == 16 || p.total >= static_cast<int64_t>(p.KB) * p.G));
  if (in_kernel) {
    auto k = block ? gemm_decode_kernel<NX, kDecodeStages, true, kSumsKernel, 0, MINB>
                   : gemm_decode_kernel<NX, kDecodeStages, false, kSumsKernel, 0, MINB>;
    if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
    return launch(k, dim3(p.G), dim3(192), L::kBytes, stream, tw, tx, p);
  }
  auto k = block ? gemm_decode_kernel<NX, kDecodeStages, true, kSumsSeparate, 0, MINB>
                 : gemm_decode_kernel<NX, kDecodeStages, false, kSumsSeparate, 0, MINB>;
  if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
  if ((st = launch(k, dim3(p.G), dim3(192), L::kBytes, stream, tw, tx, p)) != FP8Q_OK) return st;
  auto r = block ? fp8q::decode::decode_reduce_kernel<true> : fp8q::decode::decode_reduce_kernel<false>;
  return launch(r, dim3(p.n_tiles, p.M), dim3(128), 0, stream, p, NX);
}

// Weight-only FP8 on the tensor cores (2 <= M <= 64): the decode schedule
// with bf16 activations and widened weights.  Stages: 52 / 56 / 64 KB each.
template <int NX>
constexpr int w16_stages() { return NX == 64 ? 3 : 4; }

// Widen warps: 4 by default (measured: 86 us against 90 us with 8 on a 235 MB
// weight at M = 8); FP8Q_W16_WIDEN=8 selects eight (read once).
int w16_widen_warps() {
  static int n = [] {
    const char* e = getenv("FP8Q_W16_WIDEN");
    return (e && strcmp(e, "8") == 0) ? 8 : 4;
  }();
  return n;
}

template <int NX, int WIDEN>
fp8q_status launch_decode_w16_n(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int dev,
                                void* stream) {
  constexpr int kStages = w16_stages<NX>();
  using L = fp8q::decode::Layout<NX, kStages, WIDEN>;
  auto k = fp8q::decode::gemm_decode_kernel<NX, kStages, false, fp8q::decode::kSumsKernel, WIDEN>;
  fp8q_status st;
  if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
  return launch(k, dim3(p.G), dim3(L::kThreads), L::kBytes, stream, tw, tx, p);
}

template <int NX>
fp8q_status launch_decode_w16(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int dev, void* stream) {
  return w16_widen_warps() == 4 ? launch_decode_w16_n<NX, 4>(tw, tx, p, dev, stream)
                                : launch_decode_w16_n<NX, 8>(tw, tx, p, dev, stream);
}

// Weight-only kernel choice: the CUDA-core kernel for one token, the tensor
// cores above.  FP8Q_W8A16_KERNEL=cuda|tc forces one (read once; "cuda"
// applies up to 16 tokens), for comparing them on the same problem.
int w8a16_choice() {
  static int choice = [] {
    const char* e = getenv("FP8Q_W8A16_KERNEL");
    if (e && strcmp(e, "cuda") == 0) return 1;
    if (e && strcmp(e, "tc") == 0) return 2;
    return 0;
  }();
  return choice;
}

bool w8a16_uses_cuda_cores(int64_t M) {
  const int c = w8a16_choice();
  if (c == 1) return M <= fp8q::wonly::kMaxTokens;
  if (c == 2) return false;
  return M == 1;
}

// Weight-only FP8 (small M): MT padded tokens, R channels per CTA, STAGES
// shared-memory stages, MINB CTAs per SM for the register budget.
template <int MT, int R, int STAGES, int MINB>
fp8q_status launch_w8a16(const fp8q::wonly::Params& p, int dev, void* stream) {
  using L = fp8q::wonly::Layout<R, STAGES>;
  constexpr int kBytes = L::template bytes<R * MT>();
  auto k = fp8q::wonly::gemv_w8a16_kernel<MT, R, STAGES, MINB>;
  fp8q_status st;
  if ((st = ensure_smem(k, kBytes, dev)) != FP8Q_OK) return st;
  return launch(k, dim3((p.N + R - 1) / R), dim3(fp8q::wonly::kThreads), kBytes, stream, p);
}

// CTA pairs resident at once for the pair prefill kernels (block or channel
// scales), per device; computed once (a race between host threads computes
// the same value twice).  Also opts the kernels in to their shared memory.
fp8q_status prefill_pairs(bool block, int dev, int sms, int* out) {
  using L = fp8q::prefill::PairLayout<kPairStages>;
  static std::atomic<int> max_pairs[2][kMaxDevices];
  fp8q_status st;
  if (block) {
    auto k = fp8q::prefill::gemm_block2_kernel<kPairStages>;
    if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
  } else {
    if ((st = ensure_smem(fp8q::prefill::gemm_channel2_kernel<kPairStages, false>, L::kBytes, dev)) != FP8Q_OK)
      return st;
  }
  if (max_pairs[block][dev].load(std::memory_order_relaxed) == 0) {
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2 * sms);
    qc.dynamicSmemBytes = L::kBytes;
    int n = 0;
    cudaError_t e;
    if (block) {
      // The kernel moves registers between its warpgroups; that is only
      // safe when it is launched with the register count it was built for.
      auto k = fp8q::prefill::gemm_block2_kernel<kPairStages>;
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return FP8Q_ERR_CUDA;
      if (fa.numRegs != fp8q::prefill::kBlock2LaunchRegs) return FP8Q_ERR_UNSUPPORTED;
      qc.blockDim = dim3(fp8q::prefill::kBlock2Threads);
      e = cudaOccupancyMaxActiveClusters(&n, k, &qc);
    } else {
      qc.blockDim = dim3(64 + 32 * L::kEpiWarps);
      e = cudaOccupancyMaxActiveClusters(&n, fp8q::prefill::gemm_channel2_kernel<kPairStages, false>, &qc);
    }
    if (e != cudaSuccess || n < 1) n = sms / 2;
    max_pairs[block][dev].store(n, std::memory_order_relaxed);
  }
  *out = max_pairs[block][dev].load(std::memory_order_relaxed);
  return FP8Q_OK;
}

// Stream-K for the channel pair kernel, on request (FP8Q_PREFILL_STREAMK=1,
// read once): shapes whose 256 x 256 tiles fill the pairs unevenly (the
// data-parallel schedule, its last round cut into N halves where that helps,
// keeps under 92% of the pairs busy).  Not the default: measured on the
// B200 it is slower on every such Llama shape (70B M=512 gate/up 0.67 against
// 0.74 of the FP8 peak, down 0.66 against 0.83, qkv 0.47 against 0.54; 8B
// k/v at M=8192 0.51 against 0.71).  Likely costs: pairs working on different
// K ranges no longer share operand tiles through L2 at the same time, and a
// tile cut over many pairs is summed by one pair that reads every other pair's
// 256 x 256 fp32 partial alone (a variant that kept whole rounds data-parallel
// and cut only the last round's tiles by steps was slower still).
bool prefill_streamk(int num_tiles, int pairs) {
  static bool on = [] {
    const char* e = getenv("FP8Q_PREFILL_STREAMK");
    return e && strcmp(e, "1") == 0;
  }();
  if (!on) return false;
  int full, split;
  fp8q::prefill::tail_split(num_tiles, pairs, &full, &split);
  const int rest = num_tiles - full;
  const double rounds = full / static_cast<double>(pairs) +
                        (rest ? (split == 2 ? 0.5 * ((2 * rest + pairs - 1) / pairs) : (rest + pairs - 1) / pairs) : 0);
  return num_tiles / (rounds * pairs) < 0.92;
}

// Stream-K workspace: [num_tiles][2][8] arrival counters (padded to 256 bytes),
// then 2 fp32 256 x 256 partial tiles per pair.
size_t prefill_sk_counter_bytes(int num_tiles) {
  return (static_cast<size_t>(num_tiles) * 16 * sizeof(unsigned) + 255) & ~size_t(255);
}
size_t prefill_sk_bytes(int num_tiles, int pairs) {
  return prefill_sk_counter_bytes(num_tiles) +
         static_cast<size_t>(2 * pairs) * fp8q::prefill::kSkSlotFloats * sizeof(float);
}

}  // namespace

extern "C" {

fp8q_status fp8_quant_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, int mode, uint8_t* Wq,
                             int64_t ldwq, float* w_scale, void* stream) {
  fp8q_status st = check_quant_args(W_bf16, N, K, ldw, mode, Wq, ldwq, w_scale);
  if (st != FP8Q_OK || N == 0) return st;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  const uint16_t* w = static_cast<const uint16_t*>(W_bf16);
  const bool s16 = (mode & FP8Q_SCALE_BF16) != 0;
  mode &= ~FP8Q_SCALE_BF16;
  if (mode == FP8Q_CHANNEL_TOKEN)
    return launch_rows(w, N, static_cast<int>(K), ldw, Wq, ldwq, w_scale, s16, stream);
  const int64_t NB = (N + 127) / 128;
  if (NB > 65535) return FP8Q_ERR_UNSUPPORTED;
  return launch(fp8q::quant_blocks128_kernel, dim3(static_cast<unsigned>(K / 128), static_cast<unsigned>(NB)),
                dim3(256), 0, stream, w, N, static_cast<int>(K / 128), ldw, Wq, ldwq, w_scale, s16);
}

fp8q_status fp8_quant_act(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, int mode, uint8_t* Xq,
                          int64_t ldxq, float* x_scale, void* stream) {
  fp8q_status st = check_quant_args(X_bf16, M, K, ldx, mode, Xq, ldxq, x_scale);
  if (st != FP8Q_OK || M == 0) return st;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  const uint16_t* x = static_cast<const uint16_t*>(X_bf16);
  const bool s16 = (mode & FP8Q_SCALE_BF16) != 0;
  mode &= ~FP8Q_SCALE_BF16;
  if (mode == FP8Q_CHANNEL_TOKEN)
    return launch_rows(x, M, static_cast<int>(K), ldx, Xq, ldxq, x_scale, s16, stream);
  const int G = static_cast<int>(K / 128);
  const int64_t total = M * G;
  if (total >= (static_cast<int64_t>(1) << 31)) return FP8Q_ERR_UNSUPPORTED;   // 32-bit group walk
  // Groups per half warp: 4, or 6 or 8 where that lets one pass of the
  // resident CTAs (8 of 256 threads per SM) cover every group, so that no half
  // warp waits on a second DRAM round trip.
  const int64_t resident = static_cast<int64_t>(sms) * 8;
  int gpt = 4;
  if ((total + 63) / 64 > resident) gpt = (total + 95) / 96 <= resident ? 6 : 8;
  int64_t grid = (total + 16 * gpt - 1) / (16 * gpt);
  if (grid > resident) grid = resident;
  const dim3 g1(static_cast<unsigned>(grid));
  if (gpt == 4)
    return launch(fp8q::quant_groups128_kernel<4>, g1, dim3(256), 0, stream, x, M, G, ldx, Xq, ldxq, x_scale, s16);
  if (gpt == 6)
    return launch(fp8q::quant_groups128_kernel<6>, g1, dim3(256), 0, stream, x, M, G, ldx, Xq, ldxq, x_scale, s16);
  return launch(fp8q::quant_groups128_kernel<8>, g1, dim3(256), 0, stream, x, M, G, ldx, Xq, ldxq, x_scale, s16);
}

fp8q_status fp8_rmsnorm_quant_act(const void* X_bf16, const void* gamma_bf16, int64_t M, int64_t K, int64_t ldx,
                                  float eps, uint8_t* Xq, int64_t ldxq, float* x_scale, float* rstd, void* stream) {
  fp8q_status st = check_quant_args(X_bf16, M, K, ldx, FP8Q_CHANNEL_TOKEN, Xq, ldxq, x_scale);
  if (st != FP8Q_OK) return st;
  if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return FP8Q_ERR_INVALID_ARG;   // also rejects NaN
  if (M == 0) return FP8Q_OK;
  if (!gamma_bf16) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(gamma_bf16, 16) || (rstd && !aligned(rstd, 4))) return FP8Q_ERR_MISALIGNED;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  return launch_rmsnorm_rows(static_cast<const uint16_t*>(X_bf16), static_cast<const uint16_t*>(gamma_bf16), M,
                             static_cast<int>(K), ldx, eps, Xq, ldxq, x_scale, rstd, stream);
}

fp8q_status fp8_quant_act_static(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, float scale, uint8_t* Xq,
                                 int64_t ldxq, float* x_scale, void* stream) {
  if (!(scale > 0.0f) || !(scale < 3.0e38f)) return FP8Q_ERR_INVALID_ARG;   // also rejects NaN
  if (M < 0 || K <= 0 || ldx < K || ldxq < K || K % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!X_bf16 || !Xq) return FP8Q_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || ldxq % 16 != 0) return FP8Q_ERR_MISALIGNED;
  if (!aligned(X_bf16, 16) || !aligned(Xq, 16) || (x_scale && !aligned(x_scale, 4))) return FP8Q_ERR_MISALIGNED;
  if (M > kInt32Max || K > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  fp8q_status st;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  const int64_t vecs = M * (K / 8);
  if (vecs >= (static_cast<int64_t>(1) << 31)) return FP8Q_ERR_UNSUPPORTED;   // 32-bit positions
  int64_t grid = (vecs + 1023) / 1024;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  return launch(fp8q::quant_static_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, stream,
                static_cast<const uint16_t*>(X_bf16), M, static_cast<int>(K), ldx, scale, Xq, ldxq, x_scale);
}

fp8q_status fp8_calibrate_static_scale(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double lo, double hi,
                                       uint32_t* hist, float* scale, void* stream) {
  if (M <= 0 || K <= 0 || ldx < K || K % 8 != 0) return FP8Q_ERR_INVALID_ARG;
  if (!(lo >= 0.0 && lo <= 1.0) || !(hi >= 0.0 && hi <= 1.0)) return FP8Q_ERR_INVALID_ARG;   // rejects NaN
  if (!X_bf16 || !hist || !scale) return FP8Q_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(X_bf16, 16) || !aligned(hist, 4) || !aligned(scale, 4)) return FP8Q_ERR_MISALIGNED;
  if (M > kInt32Max || K > kInt32Max || M * K >= (static_cast<int64_t>(1) << 32)) return FP8Q_ERR_UNSUPPORTED;
  fp8q_status st;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  const int64_t vecs = M * (K / 8);
  int64_t grid = (vecs + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  if ((st = launch(fp8q::calib::hist_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, stream,
                   static_cast<const uint16_t*>(X_bf16), M, static_cast<int>(K), ldx, hist)) != FP8Q_OK)
    return st;
  return launch(fp8q::calib::select_kernel, dim3(1), dim3(1024), 0, stream, hist, M * K, lo, hi, scale);
}

size_t fp8_linear_workspace_size(int64_t M, int64_t N, int64_t K, int mode) {
  if (!valid_mode(mode)) return 0;
  mode &= ~FP8Q_SCALE_BF16;
  if (M <= 0 || N <= 0 || K <= 0 || M > kInt32Max || N > kInt32Max || K > kInt32Max) return 0;
  int dev, sms;
  if (current_device(&dev, &sms) != FP8Q_OK) return 0;
  if (M > kDecodeMaxM) {            // prefill: the stream-K schedule's scratch, where it pays
    const bool pair = prefill_choice() != 1 && (M >= 256 || prefill_choice() == 2);
    if (!pair || mode == FP8Q_BLOCK128) return 0;
    int pairs = 0;
    if (prefill_pairs(false, dev, sms, &pairs) != FP8Q_OK) return 0;
    const int num_tiles = static_cast<int>(((M + 255) / 256) * ((N + 255) / 256));
    const int64_t steps = static_cast<int64_t>(num_tiles) * ((K + 127) / 128);
    if (steps > kInt32Max || !prefill_streamk(num_tiles, pairs)) return 0;
    return prefill_sk_bytes(num_tiles, pairs);
  }
  int n_tiles, G, nx;
  int64_t total;
  decode_shape(M, N, K, sms, decode_half_stages(decode_nx(M)), &n_tiles, &total, &G, &nx);
  return decode_workspace_bytes(n_tiles, G, nx);
}

fp8q_status fp8_linear(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale, int64_t M,
                       int64_t N, int64_t K, int mode, void* Y_bf16, int64_t ldy, void* workspace,
                       size_t workspace_bytes, void* stream) {
  fp8q_status st = check_linear_args(Xq, x_scale, Wq, w_scale, M, N, K, mode, Y_bf16, ldy);
  if (st != FP8Q_OK || M == 0) return st;
  mode &= ~FP8Q_SCALE_BF16;                     // the scale option concerns quantization only
  if (M <= kDecodeMaxM) {                       // its size needs the device; presence and alignment do not
    if (!workspace) return FP8Q_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return FP8Q_ERR_MISALIGNED;
  }
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  const int KB = static_cast<int>((K + 127) / 128);

  if (M <= kDecodeMaxM) {
    int n_tiles, G, nx;
    int64_t total;
    decode_shape(M, N, K, sms, decode_half_stages(decode_nx(M)), &n_tiles, &total, &G, &nx);
    if (!workspace || workspace_bytes < decode_workspace_bytes(n_tiles, G, nx)) return FP8Q_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return FP8Q_ERR_MISALIGNED;
    CUtensorMap tw, tx;
    if ((st = tmap_u8_sw128(&tw, Wq, N, K, K, 128)) != FP8Q_OK) return st;
    if ((st = tmap_u8_sw128(&tx, Xq, M, K, K, static_cast<uint32_t>(nx))) != FP8Q_OK) return st;
    Params p{};
    p.early = decode_early(total, G, KB) ? 1 : 0;
    p.xs = x_scale;
    p.ws = w_scale;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.KB = KB;
    p.n_tiles = n_tiles;
    if (total > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
    p.total = static_cast<int>(total);
    p.G = G;
    decode_bind_workspace(p, workspace, Y_bf16, ldy);
    if (nx == 16) return launch_decode_nx<16>(tw, tx, p, mode, dev, sms, stream);
    if (nx == 32) return launch_decode_nx<32>(tw, tx, p, mode, dev, sms, stream);
    return launch_decode_nx<64>(tw, tx, p, mode, dev, sms, stream);
  }

  const bool pair = prefill_choice() != 1 && (M >= 256 || prefill_choice() == 2);
  if (pair) {
    using L = fp8q::prefill::PairLayout<kPairStages>;
    const bool block = mode == FP8Q_BLOCK128;
    static_assert(fp8q::prefill::PairLayout<kPairStages, 4>::kBytes == L::kBytes, "one shared-memory size");
    int pairs = 0;
    if ((st = prefill_pairs(block, dev, sms, &pairs)) != FP8Q_OK) return st;
    fp8q::prefill::Params p;
    p.xs = x_scale;
    p.ws = w_scale;
    p.y = static_cast<__nv_bfloat16*>(Y_bf16);
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.ldy = ldy;
    p.KB = KB;
    p.num_m = static_cast<int>((M + 255) / 256);
    p.num_n = static_cast<int>((N + 255) / 256);
    p.num_tiles = p.num_m * p.num_n;
    p.group_m = p.num_m < 8 ? p.num_m : 8;
    CUtensorMap ta, tb, tb64, ty;
    if ((st = tmap_u8_sw128(&ta, Xq, M, K, K, 128)) != FP8Q_OK) return st;
    if ((st = tmap_u8_sw128(&tb, Wq, N, K, K, 128)) != FP8Q_OK) return st;
    if ((st = tmap_u8_sw128(&tb64, Wq, N, K, K, 64)) != FP8Q_OK) return st;
    if ((st = tmap_bf16_sw64(&ty, Y_bf16, M, N, ldy, 32)) != FP8Q_OK) return st;
    const int64_t steps = static_cast<int64_t>(p.num_tiles) * KB;
    if (!block && steps <= kInt32Max && prefill_streamk(p.num_tiles, pairs) && workspace &&
        workspace_bytes >= prefill_sk_bytes(p.num_tiles, pairs) && aligned(workspace, 16)) {
      auto k = fp8q::prefill::gemm_channel2_kernel<kPairStages, true>;
      if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
      fp8q::prefill::SkParams sk;
      sk.count = static_cast<unsigned int*>(workspace);
      sk.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + prefill_sk_counter_bytes(p.num_tiles));
      p.full = 0;
      p.split = 1;
      const int used = steps < pairs ? static_cast<int>(steps) : pairs;
      return launch(k, dim3(2 * used), dim3(64 + 32 * L::kEpiWarps), L::kBytes, stream, ta, tb, tb64, ty, p, sk);
    }
    fp8q::prefill::tail_split(p.num_tiles, pairs, &p.full, &p.split);
    const int items = (p.full ? p.full : 0) + (p.num_tiles - p.full) * p.split;
    const int used = p.full ? pairs : (items < pairs ? items : pairs);
    if (block) {
      auto k = fp8q::prefill::gemm_block2_kernel<kPairStages>;
      return launch(k, dim3(2 * used), dim3(fp8q::prefill::kBlock2Threads), L::kBytes, stream, ta, tb, tb64, ty, p);
    }
    auto k = fp8q::prefill::gemm_channel2_kernel<kPairStages, false>;
    return launch(k, dim3(2 * used), dim3(64 + 32 * L::kEpiWarps), L::kBytes, stream, ta, tb, tb64, ty, p,
                  fp8q::prefill::SkParams{nullptr, nullptr});
  }

  fp8q::prefill::Params p;
  p.xs = x_scale;
  p.ws = w_scale;
  p.y = static_cast<__nv_bfloat16*>(Y_bf16);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ldy = ldy;
  p.KB = KB;
  const int BN = mode == FP8Q_BLOCK128 ? 128 : kPrefillBN;
  p.num_m = static_cast<int>((M + 127) / 128);
  p.num_n = static_cast<int>((N + BN - 1) / BN);
  p.num_tiles = p.num_m * p.num_n;
  p.group_m = p.num_m < 16 ? p.num_m : 16;
  int grid = p.num_tiles < sms ? p.num_tiles : sms;
  p.full = p.num_tiles;
  p.split = 1;
  if (mode != FP8Q_BLOCK128) {
    fp8q::prefill::tail_split(p.num_tiles, sms, &p.full, &p.split);
    const int items = p.full + (p.num_tiles - p.full) * p.split;
    grid = p.full ? sms : (items < sms ? items : sms);
  }
  CUtensorMap ta, tb;
  if ((st = tmap_u8_sw128(&ta, Xq, M, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tb, Wq, N, K, K, static_cast<uint32_t>(BN))) != FP8Q_OK) return st;
  if (mode == FP8Q_BLOCK128) {
    using L = fp8q::prefill::BlockLayout<kBlockStages>;
    auto k = fp8q::prefill::gemm_block_kernel<kBlockStages>;
    CUtensorMap ty;
    if ((st = tmap_bf16_sw64(&ty, Y_bf16, M, N, ldy, 32)) != FP8Q_OK) return st;
    if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
    return launch(k, dim3(grid), dim3(64 + 32 * L::kEpiWarps), L::kBytes, stream, ta, tb, ty, p);
  }
  using L = fp8q::prefill::ChannelLayout<kPrefillBN, kPrefillStages>;
  auto k = fp8q::prefill::gemm_channel_kernel<kPrefillBN, kPrefillStages>;
  CUtensorMap ty, tb128, tb64;
  if ((st = tmap_bf16_sw64(&ty, Y_bf16, M, N, ldy, 32)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tb128, Wq, N, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tb64, Wq, N, K, K, 64)) != FP8Q_OK) return st;
  if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
  return launch(k, dim3(grid), dim3(192), L::kBytes, stream, ta, tb, tb128, tb64, ty, p);
}

fp8q_status fp8_linear_swiglu(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq_gate,
                              const float* w_scale_gate, const uint8_t* Wq_up, const float* w_scale_up, int64_t M,
                              int64_t N, int64_t K, void* Y_bf16, int64_t ldy, void* stream) {
  fp8q_status st = check_linear_args(Xq, x_scale, Wq_gate, w_scale_gate, M, N, K, FP8Q_CHANNEL_TOKEN, Y_bf16, ldy);
  if (st != FP8Q_OK || M == 0) return st;
  if (!Wq_up || !w_scale_up) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(Wq_up, 16) || !aligned(w_scale_up, 4)) return FP8Q_ERR_MISALIGNED;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  using L = fp8q::prefill::PairLayout<kPairStages>;
  auto k = fp8q::prefill::gemm_swiglu2_kernel<kPairStages>;
  if ((st = ensure_smem(k, L::kBytes, dev)) != FP8Q_OK) return st;
  static std::atomic<int> max_pairs[kMaxDevices];
  if (max_pairs[dev].load(std::memory_order_relaxed) == 0) {
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2 * sms);
    qc.blockDim = dim3(64 + 32 * L::kEpiWarps);
    qc.dynamicSmemBytes = L::kBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &qc) != cudaSuccess || n < 1) n = sms / 2;
    max_pairs[dev].store(n, std::memory_order_relaxed);
  }
  fp8q::prefill::Params p;
  p.xs = x_scale;
  p.ws = w_scale_gate;
  p.y = static_cast<__nv_bfloat16*>(Y_bf16);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ldy = ldy;
  p.KB = static_cast<int>((K + 127) / 128);
  p.num_m = static_cast<int>((M + 255) / 256);
  p.num_n = static_cast<int>((N + 127) / 128);              // tiles of 128 output channels
  p.num_tiles = p.num_m * p.num_n;
  p.group_m = p.num_m < 8 ? p.num_m : 8;
  const int pairs = max_pairs[dev].load(std::memory_order_relaxed);
  fp8q::prefill::tail_split(p.num_tiles, pairs, &p.full, &p.split);
  const int items = (p.full ? p.full : 0) + (p.num_tiles - p.full) * p.split;
  const int used = p.full ? pairs : (items < pairs ? items : pairs);
  CUtensorMap ta, tg, tg64, tu, tu64, ty;
  if ((st = tmap_u8_sw128(&ta, Xq, M, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tg, Wq_gate, N, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tg64, Wq_gate, N, K, K, 64)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tu, Wq_up, N, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tu64, Wq_up, N, K, K, 64)) != FP8Q_OK) return st;
  if ((st = tmap_bf16_sw64(&ty, Y_bf16, M, N, ldy, 32)) != FP8Q_OK) return st;
  return launch(k, dim3(2 * used), dim3(64 + 32 * L::kEpiWarps), L::kBytes, stream, ta, tg, tg64, tu, tu64, ty, p,
                w_scale_up);
}

size_t fp8_linear_w8a16_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || M > kDecodeMaxM || N <= 0 || K <= 0 || w8a16_uses_cuda_cores(M)) return 0;
  int dev, sms;
  if (current_device(&dev, &sms) != FP8Q_OK) return 0;
  int n_tiles, G, nx;
  int64_t total;
  decode_shape(M, N, K, sms, false, &n_tiles, &total, &G, &nx);
  return decode_workspace_bytes(n_tiles, G, nx);
}

fp8q_status fp8_linear_w8a16(const void* X_bf16, int64_t ldx, const uint8_t* Wq, const float* w_scale, int64_t M,
                             int64_t N, int64_t K, void* Y_bf16, int64_t ldy, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || K % 16 != 0 || ldx < K || ldy < N) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!X_bf16 || !Wq || !w_scale || !Y_bf16) return FP8Q_ERR_INVALID_ARG;
  if (M > kDecodeMaxM) return FP8Q_ERR_UNSUPPORTED;
  if (N > kInt32Max || K > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  if (ldx % 8 != 0 || !aligned(X_bf16, 16) || !aligned(Wq, 16) || !aligned(Y_bf16, 2) || !aligned(w_scale, 4))
    return FP8Q_ERR_MISALIGNED;
  int dev, sms;
  fp8q_status st;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  if (w8a16_uses_cuda_cores(M)) {
    fp8q::wonly::Params p;
    p.x = static_cast<const __nv_bfloat16*>(X_bf16);
    p.ldx = ldx;
    p.w = Wq;
    p.ws = w_scale;
    p.y = static_cast<__nv_bfloat16*>(Y_bf16);
    p.ldy = ldy;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    if (M == 1) return launch_w8a16<1, 8, 2, 3>(p, dev, stream);
    if (M == 2) return launch_w8a16<2, 4, 4, 2>(p, dev, stream);
    if (M <= 4) return launch_w8a16<4, 4, 4, 2>(p, dev, stream);
    if (M <= 8) return launch_w8a16<8, 4, 4, 1>(p, dev, stream);
    return launch_w8a16<16, 1, 8, 1>(p, dev, stream);
  }
  int n_tiles, G, nx;
  int64_t total;
  decode_shape(M, N, K, sms, false, &n_tiles, &total, &G, &nx);
  if (!workspace || workspace_bytes < decode_workspace_bytes(n_tiles, G, nx)) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return FP8Q_ERR_MISALIGNED;
  CUtensorMap tw, tx;
  if ((st = tmap_u8_sw128(&tw, Wq, N, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_bf16_sw128(&tx, X_bf16, M, K, ldx, static_cast<uint32_t>(nx))) != FP8Q_OK) return st;
  Params p{};
  p.early = decode_early(total, G, static_cast<int>((K + 127) / 128)) ? 1 : 0;
  p.xs = nullptr;
  p.ws = w_scale;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.KB = static_cast<int>((K + 127) / 128);
  p.n_tiles = n_tiles;
  if (total > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  p.total = static_cast<int>(total);
  p.G = G;
  decode_bind_workspace(p, workspace, Y_bf16, ldy);
  if (nx == 16) return launch_decode_w16<16>(tw, tx, p, dev, stream);
  if (nx == 32) return launch_decode_w16<32>(tw, tx, p, dev, stream);
  return launch_decode_w16<64>(tw, tx, p, dev, stream);
}

const char* fp8q_status_string(int status) {
  switch (status) {
    case FP8Q_OK: return "FP8Q_OK";
    case FP8Q_ERR_INVALID_ARG: return "FP8Q_ERR_INVALID_ARG: invalid argument";
    case FP8Q_ERR_UNSUPPORTED: return "FP8Q_ERR_UNSUPPORTED: outside what the kernels cover";
    case FP8Q_ERR_MISALIGNED: return "FP8Q_ERR_MISALIGNED: pointer or stride not 16-byte aligned";
    case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA: a CUDA call failed";
    case FP8Q_ERR_DEVICE_TIMEOUT: return "FP8Q_ERR_DEVICE_TIMEOUT: a kernel gave up waiting";
    default: return "FP8Q: unknown status";
  }
}

int fp8q_device_error(int clear) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&v, fp8q::g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fp8q::g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
    // A kernel that gave up may have left arrival counters and partial sums in
    // fp8_linear_noalloc's in-library scratch; clearing the error restores the
    // all-zero state that entry point relies on.
    if (v != 0 && noalloc_reset_current_device() != FP8Q_OK) return -1;
  }
  return v;
}

int fp8q_version(void) { return 100; }

#ifdef FP8Q_TEST_HOOKS
// Test build only (not declared in fp8q.h, absent from the product library):
// mode 1 makes the next decode launches withhold one tensor-memory slot
// release in CTA 0, mode 2 one accumulator commit, so that a wait runs out;
// 0 turns it off.
FP8Q_API int fp8q_test_withhold(int mode) {
  const int v = mode;
  return cudaMemcpyToSymbol(fp8q::g_test_withhold, &v, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif

}  // extern "C"

// ------------------------------------------------- allocation-free variant ---
//
// fp8_linear_noalloc: the small-M (M <= 64) linear with its split-K scratch in
// a fixed array that lives in the library's device image, for callers that
// cannot allocate device memory when they call (see fp8q.h).
namespace {

// Largest scratch the allocation-free entry point can use.  Every GPU that
// loads libfp8q.so reserves this much device memory until the process exits.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;   // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device.  Host code
// must not pass the symbol itself to a kernel: on the host it names a shadow
// variable, not device memory.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Zero the allocation-free scratch of the current device, if a call there has
// looked it up (a device that never ran fp8_linear_noalloc has an untouched,
// zero-filled array).  cudaMemset allocates nothing.
fp8q_status noalloc_reset_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_UNSUPPORTED;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    p = g_noalloc_ptr[dev];
  }
  if (p == nullptr) return FP8Q_OK;
  if (cudaMemset(p, 0, kNoAllocScratchBytes) != cudaSuccess) return FP8Q_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

fp8q_status noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FP8Q_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FP8Q_OK;
}

}  // namespace

extern "C" {

fp8q_status fp8_linear_noalloc(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale,
                               int64_t M, int64_t N, int64_t K, int mode, void* Y_bf16, int64_t ldy,
                               void* stream) {
  fp8q_status st = check_linear_args(Xq, x_scale, Wq, w_scale, M, N, K, mode, Y_bf16, ldy);
  if (st != FP8Q_OK || M == 0) return st;
  mode &= ~FP8Q_SCALE_BF16;                     // the scale option concerns quantization only
  if (M > kDecodeMaxM) return FP8Q_ERR_UNSUPPORTED;    // the M > 64 path of fp8_linear needs no scratch
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != FP8Q_OK) return st;
  int n_tiles, G, nx;
  int64_t total;
  decode_shape(M, N, K, sms, decode_half_stages(decode_nx(M)), &n_tiles, &total, &G, &nx);
  if (decode_workspace_bytes(n_tiles, G, nx) > kNoAllocScratchBytes) return FP8Q_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != FP8Q_OK) return st;
  CUtensorMap tw, tx;
  if ((st = tmap_u8_sw128(&tw, Wq, N, K, K, 128)) != FP8Q_OK) return st;
  if ((st = tmap_u8_sw128(&tx, Xq, M, K, K, static_cast<uint32_t>(nx))) != FP8Q_OK) return st;
  Params p{};
  p.early = decode_early(total, G, static_cast<int>((K + 127) / 128)) ? 1 : 0;
  p.xs = x_scale;
  p.ws = w_scale;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.KB = static_cast<int>((K + 127) / 128);
  p.n_tiles = n_tiles;
  if (total > kInt32Max) return FP8Q_ERR_UNSUPPORTED;
  p.total = static_cast<int>(total);
  p.G = G;
  decode_bind_workspace(p, scratch, Y_bf16, ldy);
  if (nx == 16) return launch_decode_nx<16>(tw, tx, p, mode, dev, sms, stream);
  if (nx == 32) return launch_decode_nx<32>(tw, tx, p, mode, dev, sms, stream);
  return launch_decode_nx<64>(tw, tx, p, mode, dev, sms, stream);
}

}  // extern "C"
