// tcgen05 weight-streaming GEMM for sm_100a.
//
// Swap-AB: the weight tile (128 rows x 64 K, bf16) is the MMA's A operand and
// the few activation rows (m_tile <= 256) are its B operand, so the MMA shape is
// M=128, N=m_tile and the fp32 accumulator D[weight row][activation row] lives
// in TMEM. Both operands are K-major tiles that TMA writes with 128-byte
// swizzling. Warp roles (192 threads):
//   warp 0       TMA producer (one elected lane), ring of `stages` stages
//   warp 1       TMEM owner + MMA issuer (one elected lane)
//   warps 2..5   epilogue: TMEM -> registers -> smem chunk -> fused epilogue
// Split-K across a thread-block cluster: the `splits` CTAs of one output tile
// form a cluster, each reduces its own K range into TMEM, stages the fp32
// accumulator in its shared memory, and after a cluster barrier CTA r sums rows
// [r*m/splits, (r+1)*m/splits) over all CTAs' staging through distributed shared
// memory, in rank order (deterministic), then runs the fused epilogue on them.
// Every mbarrier wait is bounded; on a timeout the CTA flags ST_TIMEOUT, lets
// its copies in flight land, frees TMEM and returns.
#include <cooperative_groups.h>

#include "gemm.cuh"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace dfl {

using namespace sm100;

constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr int kABytes = kTileN * 64 * 2;   // 16 KB weight tile per stage

__host__ __device__ inline int stage_bytes(int m_tile) { return kABytes + m_tile * 64 * 2; }

size_t gemm_tc_smem_bytes(int m_tile, int stages) { return (size_t)stages * stage_bytes(m_tile) + 1024; }

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmTcParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[kMaxStages];
  __shared__ uint64_t empty_bar[kMaxStages];
  __shared__ uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.x = ((tile * m_blocks) + mb) * splits + split; split = rank in the cluster
  int id = blockIdx.x;
  const int split = id % p.splits;
  id /= p.splits;
  const int mb = id % p.m_blocks;
  const int tile = id / p.m_blocks;
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(p.num_kb, kb0 + p.kb_per_split);
  const int nkb = kb1 - kb0;
  const int S = p.stages;
  const int sbytes = stage_bytes(p.m_tile);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  int* status = p.epi.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    s_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if (p.paired) {
      prefetch_tmap(&p.wmap[0]);
      prefetch_tmap(&p.wmap[1]);
    } else {
      prefetch_tmap(&p.wmap[seg_of_tile(p.epi, tile)]);
    }
    prefetch_tmap(&p.xmap);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0 && nkb > 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int seg = p.paired ? 0 : seg_of_tile(p.epi, tile);
      const int wrow = p.paired ? tile * (kTileN / 2) : (tile - p.epi.seg_tile_begin[seg]) * kTileN;
      const uint32_t tx = (uint32_t)sbytes;
      const int pre = min(nkb, S);
      // The first `pre` stages' weight tiles do not depend on the previous kernel:
      // issue them before waiting for it (programmatic dependent launch).
      for (int i = 0; i < pre; ++i) {
        uint8_t* a = base + (size_t)i * sbytes;
        const int kc = (kb0 + i) * 64;
        mbar_arrive_expect_tx(&full_bar[i], tx);
        if (p.paired) {
          tma_load_2d(a, &p.wmap[0], &full_bar[i], kc, wrow, pol_w);
          tma_load_2d(a + kABytes / 2, &p.wmap[1], &full_bar[i], kc, wrow, pol_w);
        } else {
          tma_load_2d(a, &p.wmap[seg], &full_bar[i], kc, wrow, pol_w);
        }
      }
      grid_dep_wait();
      for (int i = 0; i < pre; ++i)
        tma_load_2d(base + (size_t)i * sbytes + kABytes, &p.xmap, &full_bar[i], (kb0 + i) * 64, mb * p.m_tile, pol_x);
      int issued = pre;
      bool ok = true;
      for (int i = pre; i < nkb && ok; ++i) {
        const int s = i % S;
        ok = mbar_wait(&empty_bar[s], ((i / S) & 1) ^ 1, status);
        if (!ok) break;
        uint8_t* a = base + (size_t)s * sbytes;
        uint8_t* b = a + kABytes;
        const int kc = (kb0 + i) * 64;
        mbar_arrive_expect_tx(&full_bar[s], tx);
        if (p.paired) {
          tma_load_2d(a, &p.wmap[0], &full_bar[s], kc, wrow, pol_w);
          tma_load_2d(a + kABytes / 2, &p.wmap[1], &full_bar[s], kc, wrow, pol_w);
        } else {
          tma_load_2d(a, &p.wmap[seg], &full_bar[s], kc, wrow, pol_w);
        }
        tma_load_2d(b, &p.xmap, &full_bar[s], kc, mb * p.m_tile, pol_x);
        ++issued;
      }
      grid_dep_launch();
      // Let every copy this CTA issued land before the CTA can exit.
      for (int i = max(0, issued - S); i < issued; ++i) mbar_wait(&full_bar[i % S], (i / S) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0 && nkb > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.m_tile);
      bool ok = true;
      int i = 0;
      for (; i < nkb; ++i) {
        const int s = i % S;
        ok = mbar_wait(&full_bar[s], (i / S) & 1, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_addr(base + (size_t)s * sbytes);
        const uint32_t b = a + kABytes;
        const uint64_t ad = desc_kmajor_sw128(a), bd = desc_kmajor_sw128(b);
#pragma unroll
        for (int k = 0; k < 4; ++k)  // 4 x K=16 per 64-wide stage; +32 B per step inside the swizzle atom
          mma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (i | k) != 0 ? 1u : 0u);
        mma_commit(&empty_bar[s]);
      }
      if (!ok) s_flag = 1;
      mma_commit(&acc_bar);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int t = q * 32 + lane;           // tile row owned by this thread
    const int row0 = mb * p.m_tile;
    const int rows_here = min(p.m_tile, p.M - row0);
    float* chunk = reinterpret_cast<float*>(base);
    grid_dep_wait();   // epilogue reads / writes data shared with the previous kernel
    bool ok = nkb > 0 ? mbar_wait(&acc_bar, 0, status) : true;
    if (!ok) s_flag = 1;
    named_bar_sync(1, 128);
    ok = (s_flag == 0) && nkb > 0;
    tc_fence_after();
    grid_dep_launch();
    if (ok) {
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
      float v[32];
      if (p.splits == 1) {
        for (int c0 = 0; c0 < rows_here; c0 += kChunkRows) {
          tmem_ld_32x32b_x32(lane_base + (uint32_t)c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) chunk[j * kChunkLd + t] = v[j];
          named_bar_sync(1, 128);
          epilogue_chunk(p.epi, tile, row0 + c0, min(kChunkRows, rows_here - c0), chunk, t);
          named_bar_sync(1, 128);
        }
      } else {
        // stage this split's accumulator: stage[m][t], m < rows_here
        float* stage = reinterpret_cast<float*>(base);
        for (int c0 = 0; c0 < rows_here; c0 += kChunkRows) {
          tmem_ld_32x32b_x32(lane_base + (uint32_t)c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < rows_here) stage[(c0 + j) * kTileN + t] = v[j];
        }
      }
    } else if (p.splits > 1) {
      // no K range (or a timed-out wait): contribute zeros
      float* stage = reinterpret_cast<float*>(base);
      for (int m = 0; m < rows_here; ++m) stage[m * kTileN + t] = 0.f;
    }
    tc_fence_before();
  }
  if (p.splits > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();   // every split's staging is written
    if (warp >= 2) {
      const int t = (warp & 3) * 32 + lane;
      const int row0 = mb * p.m_tile;
      const int rows_here = min(p.m_tile, p.M - row0);
      const int per = (rows_here + p.splits - 1) / p.splits;
      const int r_lo = split * per, r_hi = min(rows_here, r_lo + per);
      float* stage = reinterpret_cast<float*>(base);
      float* chunk = stage + (size_t)p.m_tile * kTileN;
      const float* rem[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) rem[s] = s < p.splits ? cluster.map_shared_rank(stage, s) : stage;
      for (int c0 = r_lo; c0 < r_hi; c0 += kChunkRows) {
        const int nr = min(kChunkRows, r_hi - c0);
        for (int j = 0; j < nr; ++j) {
          const int off = (c0 + j) * kTileN + t;
          float part[8];
#pragma unroll
          for (int s = 0; s < 8; ++s) part[s] = s < p.splits ? rem[s][off] : 0.f;
          float sum = 0.f;
#pragma unroll
          for (int s = 0; s < 8; ++s) sum += part[s];
          chunk[j * kChunkLd + t] = sum;
        }
        named_bar_sync(1, 128);
        epilogue_chunk(p.epi, tile, row0 + c0, nr, chunk, t);
        named_bar_sync(1, 128);
      }
    }
    cluster.sync();   // no CTA leaves while a peer may still read its staging
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
  }
}

int gemm_tc_max_active_clusters(int m_tile, int stages, int splits) {
  const size_t smem = gemm_tc_smem_bytes(m_tile, stages);
  static size_t attr_bytes_q = 0;
  if (smem > attr_bytes_q) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return 0;
    attr_bytes_q = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)splits * 64);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_gemm_tc(const GemmTcParams& p, cudaStream_t st) {
  const size_t smem = gemm_tc_smem_bytes(p.m_tile, p.stages);
  // the opt-in limit covers static + dynamic shared memory: raise the dynamic
  // limit only as far as this launch needs
  static size_t attr_bytes = 0;
  if (smem > attr_bytes) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.n_tiles * p.splits * p.m_blocks));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = p.use_pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.splits > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel, p);
}

}  // namespace dfl
