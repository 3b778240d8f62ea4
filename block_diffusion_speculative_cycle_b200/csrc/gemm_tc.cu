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
// form a cluster and each reduces its own K range into TMEM. Rows of the tile
// are owned in blocks of `per` by the cluster's CTAs: every CTA stages its fp32
// partial rows in its own shared memory and bulk-copies each owner's block into
// the owner's receive buffer (distributed shared memory, counted on the owner's
// mbarrier); the owner waits for exactly the bytes it expects, sums the splits
// in rank order (deterministic) and runs the fused epilogue on its rows.
// Every mbarrier wait is bounded; on a timeout the CTA flags ST_TIMEOUT, lets
// its copies in flight land, frees TMEM and returns.
#include "gemm.cuh"
#include "sm100.cuh"


namespace dfl {

using namespace sm100;

constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr int kABytes = kTileN * 64 * 2;   // 16 KB weight tile per stage

__host__ __device__ inline int stage_bytes(int m_tile, int x_split) { return kABytes + (1 + x_split) * m_tile * 64 * 2; }

// receive buffer of the cluster reduction: splits x per x 128 fp32, per = ceil(m_tile / splits)
__host__ __device__ inline size_t recv_bytes(int m_tile, int splits) {
  return splits > 1 ? (size_t)splits * ((m_tile + splits - 1) / splits) * kTileN * 4 : 0;
}

size_t gemm_tc_smem_bytes(int m_tile, int x_split, int stages, int splits) {
  return (size_t)stages * stage_bytes(m_tile, x_split) + recv_bytes(m_tile, splits) + 1024;
}

// One instantiation per epilogue kind, so a CTA fetches only its own epilogue's code.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 3) gemm_tc_kernel(const __grid_constant__ GemmTcParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[kMaxStages];
  __shared__ uint64_t empty_bar[kMaxStages];
  __shared__ uint64_t acc_bar;
  __shared__ uint64_t recv_bar;
  __shared__ uint64_t stall_bar;   // failure-injection hook only: never arrived at
  __shared__ uint32_t tmem_slot;
  __shared__ int s_flag;
  __shared__ __align__(16) float epi_scratch[kEpiScratch];
  __shared__ float row_scale[256];   // deferred-norm scales of the tile's activation rows

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
  const int sbytes = stage_bytes(p.m_tile, p.x_split);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  float* recv = reinterpret_cast<float*>(base + (size_t)S * sbytes);   // [splits][per][128]
  int* status = p.epi.status;
  const int row0 = mb * p.m_tile;
  const int rows_here = min(p.m_tile, p.M - row0);
  const int per = (p.m_tile + p.splits - 1) / p.splits;
  const int own_lo = min(rows_here, split * per), own_hi = min(rows_here, own_lo + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    mbar_init(&recv_bar, 1);
    mbar_init(&stall_bar, 1);
    s_flag = 0;
    fence_mbar_init();
    if (p.splits > 1) mbar_arrive_expect_tx(&recv_bar, (uint32_t)(p.splits * (own_hi - own_lo) * kTileN * 4));
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
  // every CTA's receive barrier is initialised before any peer may push into it
  if (p.splits > 1) cluster_arrive_release();

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
      for (int i = 0; i < pre; ++i) {
        uint8_t* b = base + (size_t)i * sbytes + kABytes;
        tma_load_2d(b, &p.xmap, &full_bar[i], (kb0 + i) * 64, mb * p.m_tile, pol_x);
        if (p.x_split)
          tma_load_2d(b + p.m_tile * 128, &p.xmap, &full_bar[i], (kb0 + i) * 64, p.x_plane_rows + mb * p.m_tile, pol_x);
      }
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
        if (p.x_split) tma_load_2d(b + p.m_tile * 128, &p.xmap, &full_bar[s], kc, p.x_plane_rows + mb * p.m_tile, pol_x);
        ++issued;
      }
      grid_dep_launch();
      // Let every copy this CTA issued land before the CTA can exit.
      for (int i = max(0, issued - S); i < issued; ++i) mbar_wait(&full_bar[i % S], (i / S) & 1, status);
    }
  } else if (warp == 1) {
    if (lane == 0 && nkb > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, (1 + p.x_split) * p.m_tile);
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
    float* chunk = reinterpret_cast<float*>(base);   // the ring is free once the accumulator is final
    grid_dep_wait();   // epilogue reads / writes data shared with the previous kernel
    // the row scales depend only on earlier kernels: compute them while the MMAs run
    epilogue_row_scales(p.epi, row0, rows_here, row_scale, t);
    // side job, also in the MMAs' shadow: this CTA's share of the next launch's RoPE table
    rope_fill_range(p.epi.fill, (int)blockIdx.x * 128 + t, (int)gridDim.x * 128);
    bool got = nkb > 0 ? mbar_wait(&acc_bar, 0, status) : true;
    // failure-injection hook: a wait that can only run out (nothing is in flight now)
    if (p.test_stall_ns && got) got = mbar_wait(&stall_bar, 0, status, p.test_stall_ns);
    // one decision for all 128 threads (the MMA lane may set s_flag at any time)
    bool ok = !named_bar_or(1, 128, !got || s_flag != 0) && nkb > 0;
    tc_fence_after();
    grid_dep_launch();
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    float v[32];
    // rows c0 .. c0+31 of this thread's tile row: the hi-plane accumulator plus,
    // with split activations, the lo-plane one m_tile columns further on
    auto load_rows = [&](int c0) {
      tmem_ld_32x32b_x32(lane_base + (uint32_t)c0, v);
      if (p.x_split) {
        float w[32];
        tmem_ld_32x32b_x32(lane_base + (uint32_t)(p.m_tile + c0), w);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += w[j];
      }
    };
    if (p.splits == 1) {
      if (ok) {
        for (int c0 = 0; c0 < rows_here; c0 += kChunkRows) {
          load_rows(c0);
#pragma unroll
          for (int j = 0; j < 32; ++j) chunk[j * kChunkLd + t] = v[j];
          named_bar_sync(1, 128);
          epilogue_chunk_k<KIND>(p.epi, tile, row0 + c0, min(kChunkRows, rows_here - c0), chunk, t, row_scale + c0,
                                 epi_scratch + kChunkRows);
          named_bar_sync(1, 128);
        }
      }
    } else {
      // stage this split's partial rows (zeros if there was nothing to add) in the
      // ring's memory, then bulk-copy each owner's block of rows into its receive buffer
      cluster_wait_acquire();
      float* stage = reinterpret_cast<float*>(base);   // [rows_here][128]
      for (int c0 = 0; c0 < rows_here; c0 += kChunkRows) {
        if (ok) {
          load_rows(c0);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < rows_here) stage[(c0 + j) * kTileN + t] = v[j];
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (t == 0) {
        const uint32_t recv_s = smem_addr(recv), bar_s = smem_addr(&recv_bar), stage_s = smem_addr(stage);
        for (int k = 0; k < p.splits; ++k) {
          const int lo = min(rows_here, k * per), hi = min(rows_here, lo + per);
          if (hi > lo)
            bulk_copy_s2s(mapa_shared(recv_s + (uint32_t)(split * per * kTileN * 4), (uint32_t)k),
                          stage_s + (uint32_t)(lo * kTileN * 4), (uint32_t)((hi - lo) * kTileN * 4),
                          mapa_shared(bar_s, (uint32_t)k));
        }
        bulk_commit();
      }
      // receive: all splits' partials of the rows this CTA owns, then sum in split order
      chunk = stage + (size_t)rows_here * kTileN;   // outgoing copies may still read the staging
      const bool got = mbar_wait(&recv_bar, 0, status);
      for (int c0 = own_lo; got && c0 < own_hi; c0 += kChunkRows) {
        const int nr = min(kChunkRows, own_hi - c0);
        for (int j = 0; j < nr; ++j) {
          const int rl = c0 - own_lo + j;
          float sum = 0.f;
          for (int sp = 0; sp < p.splits; ++sp) sum += recv[(sp * per + rl) * kTileN + t];
          chunk[j * kChunkLd + t] = sum;
        }
        named_bar_sync(1, 128);
        epilogue_chunk_k<KIND>(p.epi, tile, row0 + c0, nr, chunk, t, row_scale + c0, epi_scratch + kChunkRows);
        named_bar_sync(1, 128);
      }
      if (t == 0) bulk_wait_read_all();   // this CTA's staging has been read by every copy
    }
    tc_fence_before();
  }
  // producer and MMA threads pass the cluster barrier they arrived at (epilogue threads already did)
  if (p.splits > 1 && warp < 2) cluster_wait_acquire();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
  }
}

cudaError_t launch_gemm_tc(const GemmTcParams& p, cudaStream_t st) {
  const size_t smem = gemm_tc_smem_bytes(p.m_tile, p.x_split, p.stages, p.splits);
  // the opt-in limit covers static + dynamic shared memory: raise the dynamic
  // limit only as far as this launch needs
  const void* kernel = nullptr;
  switch (p.epi.kind) {
    case EPI_STORE: kernel = (const void*)gemm_tc_kernel<EPI_STORE>; break;
    case EPI_QKV: kernel = (const void*)gemm_tc_kernel<EPI_QKV>; break;
    case EPI_KV_INJECT: kernel = (const void*)gemm_tc_kernel<EPI_KV_INJECT>; break;
    case EPI_RESID: kernel = (const void*)gemm_tc_kernel<EPI_RESID>; break;
    case EPI_SWIGLU: kernel = (const void*)gemm_tc_kernel<EPI_SWIGLU>; break;
    case EPI_ARGMAX: kernel = (const void*)gemm_tc_kernel<EPI_ARGMAX>; break;
    case EPI_SAMPLE: kernel = (const void*)gemm_tc_kernel<EPI_SAMPLE>; break;
    default: return cudaErrorInvalidValue;
  }
  static size_t attr_bytes[EPI_SAMPLE + 1] = {};
  if (smem > attr_bytes[p.epi.kind]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes[p.epi.kind] = smem;
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
  void* args[] = {const_cast<GemmTcParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, kernel, args);
}

}  // namespace dfl
