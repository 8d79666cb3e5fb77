// Dense projections on either side of the block-sparse attention, for B200 (sm_100a).
//
// The layer the pages build around the attention maps the hidden states x [B, L, C]
// to q, k and v with one linear map split into heads ("BigBird 稀疏注意力机制解析",
// 代码实现: self.qkv = nn.Linear(dim, dim * 3), then the per-head split), and maps
// the merged heads back with an output projection ("BERT 稀疏注意力机制入门指南",
// PyTorch 实现: self.proj = nn.Linear(dim, dim)).  Both are D = A W^T + bias with W
// in the [out, in] layout of a linear layer.  Here the layout changes around the
// attention are part of the GEMMs' own memory access, so no transpose runs between
// the kernels:
//   - QKV projection: A = x read as [B, L, C]; the epilogue stores each 64-column
//     group of D straight into q, k or v in the attention's [B, H, L, 64] layout.
//   - Output projection: A = the attention output O [B, H, L, 64] read through a
//     3-D tensor map, one head per 64-wide K block (the head merge happens in the
//     tile load); D is stored as y [B, L, N].
//
// Kernel: persistent, one CTA per SM, 192 threads.  A tile is 128 rows of one batch
// element by 256 output columns.
//   warp 0     TMA producer: per 64-wide K block, the A box (128 x 64) and the W box
//              (256 x 64) into a 4-stage ring of 48 KB stages (128-byte swizzle).
//   warp 1     allocates 512 TMEM columns; lane 0 issues tcgen05.mma (M = 128,
//              N = 256, K = 16; four per K block) into accumulator stage (tile % 2),
//              so a tile's epilogue overlaps the next tile's MMAs.
//   warps 2-5  epilogue: warp w drains TMEM lanes 32 (w % 4)..+31 (the tile's rows),
//              adds the bias in fp32, rounds to bf16 (RNE) and writes 32 x 64 boxes
//              by TMA store through two 4 KB staging buffers of its own.
// Every wait is bounded; on expiry the CTA records BSA_ERR_DEVICE_TIMEOUT, drains its
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "sm100_ptx.cuh"
#include "bsa_wait.cuh"
#include "bsa_host_cuda.h"

namespace bsa {
namespace {

constexpr int kPThreads = 192;
constexpr int kBM = 128;  // tile rows (TMEM lanes)
constexpr int kBN = 256;  // tile columns (TMEM columns of one accumulator stage)
constexpr int kBK = 64;   // K block: one 128-byte swizzle atom of bf16
constexpr int kPStages = 4;
constexpr uint32_t kPABytes = kBM * kBK * 2;
constexpr uint32_t kPBBytes = kBN * kBK * 2;
constexpr uint32_t kPStageBytes = kPABytes + kPBBytes;
constexpr uint32_t kPStgBytes = 32 * 128;  // one warp's 32 x 64 bf16 output box
constexpr int kEpiWarp0 = 2;
constexpr uint32_t kPSmemStg = kPStages * kPStageBytes;
constexpr uint32_t kPSmemBar = kPSmemStg + 4 * 2 * kPStgBytes;
enum : int {
  kPFull = 0,                     // [stage] the K block's A and W boxes landed (TMA)
  kPEmpty = kPFull + kPStages,    // [stage] MMA commit: the stage may be refilled
  kPAccFull = kPEmpty + kPStages,  // [acc stage] MMA commit after a tile's last K block
  kPAccEmpty = kPAccFull + 2,     // [acc stage] the four epilogue warps drained it
  kPFinal = kPAccEmpty + 2,       // the issuer's last commit, before TMEM is freed
  kPNumBars = kPFinal + 1
};
constexpr uint32_t kPSmemMisc = kPSmemBar + 8 * kPNumBars;  // u32 TMEM base, int abort flag
constexpr uint32_t kPSmemAlloc = kPSmemMisc + 16 + 1024;    // + slack for 1024-byte alignment
static_assert(kPSmemAlloc <= 227 * 1024, "shared memory budget");
static_assert(kPStageBytes % 1024 == 0 && kPABytes % 1024 == 0 && kPStgBytes % 1024 == 0,
              "swizzle atoms must stay 1024-byte aligned");
constexpr uint32_t kPTmemCols = 2 * kBN;

struct ProjParams {
  CUtensorMap tm_a;     // 3-D, box {64, 128, 1}
  CUtensorMap tm_w;     // 2-D [N, K], box {64, 256}
  CUtensorMap tm_d[3];  // 3-D destinations, box {64, 32, 1}
  const __nv_bfloat16* bias;  // [N] or null
  int L, N, nk;               // rows per batch element, output columns, K blocks
  int a_heads;  // A is O [B, H, L, 64] (K block kb = head kb); else x [B, L, K]
  int d_heads;  // D goes to q, k, v [B, H, L, 64]; else to y [B, L, N]
  int H;        // heads of the [B, H, L, 64] side
  int C;        // d_heads: columns per destination (64 H)
  int mt_per_b, n_tiles, tiles;
  uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t pbar(uint32_t bars, int i) { return bars + 8u * static_cast<uint32_t>(i); }

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int x, int y, int z,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
// At most one of this thread's bulk stores still reads its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_le1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

struct TileCoord {
  int b, l0, n0;
};
__device__ __forceinline__ TileCoord tile_of(const ProjParams& p, int t) {
  const int bm = t / p.n_tiles;
  return TileCoord{bm / p.mt_per_b, (bm % p.mt_per_b) * kBM, (t % p.n_tiles) * kBN};
}

__device__ void producer(const ProjParams& p, uint32_t smem, uint32_t bars, volatile int* abort_flag) {
  const uint64_t pol_a = ptx::policy_evict_first(), pol_w = ptx::policy_evict_last();
  uint32_t it = 0;  // K blocks loaded so far
  bool alive = true;
  for (int t = blockIdx.x; alive && t < p.tiles; t += gridDim.x) {
    const TileCoord tc = tile_of(p, t);
    for (int kb = 0; kb < p.nk; ++kb, ++it) {
      const uint32_t s = it % kPStages;
      if (it >= kPStages &&
          !wait_one(pbar(bars, kPEmpty + s), ((it / kPStages) - 1u) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      const uint32_t full = pbar(bars, kPFull + s);
      const uint32_t dst = smem + s * kPStageBytes;
      ptx::mbar_arrive_expect_tx(full, kPStageBytes);
      if (p.a_heads)
        tma_load_3d(dst, &p.tm_a, full, 0, tc.l0, tc.b * p.H + kb, pol_a);
      else
        tma_load_3d(dst, &p.tm_a, full, kb * kBK, tc.l0, tc.b, pol_a);
      ptx::tma_load_2d(dst + kPABytes, &p.tm_w, full, kb * kBK, tc.n0, pol_w);
    }
  }
  // the last load of each stage has landed before the CTA may exit
  for (uint32_t j = it > kPStages ? it - kPStages : 0u; j < it; ++j)
    wait_force(pbar(bars, kPFull + static_cast<int>(j % kPStages)), (j / kPStages) & 1u, abort_flag,
               p.timeout_ns);
}

__device__ void mma_issuer(const ProjParams& p, uint32_t smem, uint32_t bars, uint32_t tmem,
                           volatile int* abort_flag) {
  constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, kBN, false);
  uint32_t it = 0, tcount = 0;
  bool alive = true;
  for (int t = blockIdx.x; alive && t < p.tiles; t += gridDim.x, ++tcount) {
    const uint32_t as = tcount & 1u;
    if (tcount >= 2 &&
        !wait_one(pbar(bars, kPAccEmpty + as), ((tcount >> 1) - 1u) & 1u, abort_flag, p.timeout_ns))
      break;
    ptx::tc_fence_after();
    const uint32_t d = tmem + as * kBN;
    for (int kb = 0; kb < p.nk; ++kb, ++it) {
      const uint32_t s = it % kPStages;
      if (!wait_one(pbar(bars, kPFull + s), (it / kPStages) & 1u, abort_flag, p.timeout_ns)) {
        alive = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t sa = smem + s * kPStageBytes;
      // K-major operands: each K step of 16 is +32 bytes in the descriptor's start field
      const uint64_t da = ptx::smem_desc_sw128(sa, 16), db = ptx::smem_desc_sw128(sa + kPABytes, 16);
#pragma unroll
      for (int j = 0; j < kBK / 16; ++j)
        ptx::mma_ss(d, da + 2u * j, db + 2u * j, kIdesc, (kb > 0 || j > 0) ? 1u : 0u);
      ptx::mma_commit(pbar(bars, kPEmpty + s));
    }
    if (!alive) break;
    ptx::mma_commit(pbar(bars, kPAccFull + as));
  }
  // every MMA this thread issued is done before TMEM is released
  ptx::mma_commit(pbar(bars, kPFinal));
  wait_force(pbar(bars, kPFinal), 0u, abort_flag, p.timeout_ns);
}

__device__ void epilogue(const ProjParams& p, uint32_t smem, uint8_t* smem_gen, uint32_t bars, uint32_t tmem,
                         int warp, int lane, volatile int* abort_flag) {
  const int qd = warp & 3;  // TMEM lane quadrant this warp may read
  const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
  const uint32_t stg0 = kPSmemStg + static_cast<uint32_t>(warp - kEpiWarp0) * 2u * kPStgBytes;
  uint32_t tcount = 0, sg = 0;
  for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tcount) {
    const uint32_t as = tcount & 1u;
    if (!wait_warp(pbar(bars, kPAccFull + as), (tcount >> 1) & 1u, abort_flag, p.timeout_ns)) break;
    ptx::tc_fence_after();
    const TileCoord tc = tile_of(p, t);
    const int y = tc.l0 + qd * 32;  // first row of this warp's boxes
    const uint32_t taddr = tmem + lane_addr + as * kBN;
    for (int g = 0; g < kBN / 64; ++g) {
      const int n = tc.n0 + 64 * g;
      if (n >= p.N) break;  // the last column tile may be narrower
      const uint32_t buf = stg0 + (sg & 1u) * kPStgBytes;
      if (lane == 0) bulk_wait_read_le1();  // the store that used this buffer last has read it
      __syncwarp();
      uint32_t r[2][32];
      ptx::tmem_ld32(taddr + 64u * g, r[0]);
      ptx::tmem_ld32(taddr + 64u * g + 32u, r[1]);
      ptx::tmem_wait_ld();
      ptx::reg_fence(r[0]);
      ptx::reg_fence(r[1]);
      // row `lane` of the box: 16-byte chunk j at lane * 128 + ((j ^ (lane % 8)) * 16)
      uint8_t* row = smem_gen + buf + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float bj[8];
        if (p.bias != nullptr) {
          const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + n + 8 * j));
          const uint32_t bv[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            bj[2 * c] = __uint_as_float(bv[c] << 16);
            bj[2 * c + 1] = __uint_as_float(bv[c] & 0xffff0000u);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) bj[c] = 0.f;
        }
        uint32_t w4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = 8 * j + 2 * c;
          w4[c] = pack_bf16x2(__uint_as_float(r[col >> 5][col & 31]) + bj[2 * c],
                              __uint_as_float(r[(col + 1) >> 5][(col + 1) & 31]) + bj[2 * c + 1]);
        }
        *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && y < p.L) {  // rows past L are clipped by the store; boxes wholly past it skipped
        if (p.d_heads) {
          const int which = n / p.C, h = (n % p.C) / 64;
          tma_store_3d(&p.tm_d[which], smem + buf, 0, y, tc.b * p.H + h);
        } else {
          tma_store_3d(&p.tm_d[0], smem + buf, n, y, tc.b);
        }
        ptx::bulk_commit_group();
      }
      ++sg;
    }
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(pbar(bars, kPAccEmpty + as));
  }
  if (lane == 0) ptx::bulk_wait_all();  // the stores are complete before the CTA exits
}

}  // namespace

__global__ void __launch_bounds__(kPThreads, 1) bsa_proj_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kPSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPSmemMisc + 4);
  const uint32_t bars = base + kPSmemBar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPNumBars; ++i)
      ptx::mbar_init(pbar(bars, i), (i >= kPAccEmpty && i < kPAccEmpty + 2) ? 4u : 1u);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tensormap(&p.tm_a);
    ptx::prefetch_tensormap(&p.tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(const_cast<uint32_t*>(&misc[0])), kPTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  if (warp == 0) {
    if (lane == 0) producer(p, base, bars, abort_flag);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(p, base, bars, tmem, abort_flag);
  } else {
    epilogue(p, base, smem, bars, tmem, warp, lane, abort_flag);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, kPTmemCols);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor of dims[0] (innermost, contiguous) x dims[1] (x dims[2]) elements with
// the given row and plane strides in bytes, 128-byte swizzle.
bool encode(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [planes, rows, 64] bf16 (the attention's [B, H, L, 64]), boxes of 64 x box_rows.
bool map_heads(CUtensorMap* m, const void* ptr, uint64_t planes, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[3] = {64, rows, planes};
  const cuuint64_t strides[2] = {128, rows * 128};
  const cuuint32_t box[3] = {64, box_rows, 1};
  return encode(m, ptr, 3, dims, strides, box);
}

// [B, rows, cols] bf16 row-major, boxes of 64 columns x box_rows.
bool map_rows(CUtensorMap* m, const void* ptr, uint64_t B, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const cuuint64_t dims[3] = {cols, rows, B};
  const cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  return encode(m, ptr, 3, dims, strides, box);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per device, once: whether it is an sm_100 part, its SM count, and the kernel's
// shared-memory attribute set.  A failed setup is not cached (the next call retries).
constexpr int kMaxProjDevices = 64;
int g_proj_sms[kMaxProjDevices] = {};
std::mutex g_proj_mu;

int device_sms() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxProjDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_proj_mu);
  if (g_proj_sms[dev] != 0) return g_proj_sms[dev];
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (major != 10 || minor != 0) {
    g_proj_sms[dev] = BSA_ERR_UNSUPPORTED;
    return BSA_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(bsa_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kPSmemAlloc)) != cudaSuccess)
    return BSA_ERR_CUDA;
  g_proj_sms[dev] = sms;
  return sms;
}

int launch(ProjParams& p, int B, cudaStream_t s) {
  const int sms = device_sms();
  if (sms < 0) return sms;
  p.mt_per_b = (p.L + kBM - 1) / kBM;
  p.n_tiles = (p.N + kBN - 1) / kBN;
  const long long tiles = static_cast<long long>(B) * p.mt_per_b * p.n_tiles;
  if (tiles > (1ll << 30)) return BSA_ERR_INVALID_ARG;
  p.tiles = static_cast<int>(tiles);
  p.timeout_ns = kDefaultTimeoutNs;
  const int grid = static_cast<int>(std::min<long long>(tiles, sms));
  bsa_proj_kernel<<<grid, kPThreads, kPSmemAlloc, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

}  // namespace

int proj_take_status() {
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_bsa_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_bsa_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  return st;
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_qkv_projection(const void* x, const void* w, const void* bias, int B, int L, int H, void* q, void* k,
                       void* v, void* stream) {
  if (x == nullptr || w == nullptr || q == nullptr || k == nullptr || v == nullptr) return BSA_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || H < 1 || H > (1 << 16) || static_cast<long long>(B) * H > (1ll << 30) ||
      static_cast<long long>(B) * L > (1ll << 31) - 1)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (bias != nullptr && !aligned16(bias)))
    return BSA_ERR_INVALID_ARG;
  const int C = 64 * H;
  ProjParams p{};
  if (!map_rows(&p.tm_a, x, B, L, C, kBM)) return BSA_ERR_CUDA;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(3 * C)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
    const cuuint32_t box[2] = {64, kBN};
    if (!encode(&p.tm_w, w, 2, dims, strides, box)) return BSA_ERR_CUDA;
  }
  void* dst[3] = {q, k, v};
  for (int i = 0; i < 3; ++i)
    if (!map_heads(&p.tm_d[i], dst[i], static_cast<uint64_t>(B) * H, L, 32)) return BSA_ERR_CUDA;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.L = L;
  p.N = 3 * C;
  p.nk = H;  // K = C = 64 H
  p.a_heads = 0;
  p.d_heads = 1;
  p.H = H;
  p.C = C;
  return launch(p, B, static_cast<cudaStream_t>(stream));
}

int bsa_out_projection(const void* o, const void* w, const void* bias, int B, int H, int L, int N, void* y,
                       void* stream) {
  if (o == nullptr || w == nullptr || y == nullptr) return BSA_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || H < 1 || H > (1 << 16) || N < 64 || N % 64 != 0 || N > (1 << 24) ||
      static_cast<long long>(B) * H > (1ll << 30) || static_cast<long long>(B) * L > (1ll << 31) - 1)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(w) || !aligned16(y) || (bias != nullptr && !aligned16(bias)))
    return BSA_ERR_INVALID_ARG;
  const int K = 64 * H;
  ProjParams p{};
  if (!map_heads(&p.tm_a, o, static_cast<uint64_t>(B) * H, L, kBM)) return BSA_ERR_CUDA;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, kBN};
    if (!encode(&p.tm_w, w, 2, dims, strides, box)) return BSA_ERR_CUDA;
  }
  if (!map_rows(&p.tm_d[0], y, B, L, N, 32)) return BSA_ERR_CUDA;
  p.tm_d[1] = p.tm_d[0];
  p.tm_d[2] = p.tm_d[0];
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.L = L;
  p.N = N;
  p.nk = H;  // one head per K block
  p.a_heads = 1;
  p.d_heads = 0;
  p.H = H;
  p.C = N;
  return launch(p, B, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
