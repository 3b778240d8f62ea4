// CUDA-core GEMM for the fp32 drafter (tcgen05 has no fp32 operand kind, and
// tf32 would miss the fp32 accuracy bar). Same tiling contract and fused
// epilogues as the tensor-core kernel: one CTA computes 32 activation rows x
// 128 weight rows with the full K reduction, stages the tile in shared memory
// and applies epilogue_chunk.
#include "gemm.cuh"

namespace dfl {

constexpr int kKT = 32;

template <typename WT, typename XT>
__global__ void __launch_bounds__(128) gemm_simt_kernel(const GemmSimtParams p) {
  __shared__ float xs[kChunkRows][kKT + 1];
  __shared__ float ws[kTileN][kKT + 1];
  __shared__ float chunk[kChunkRows * kChunkLd];
  __shared__ __align__(16) float epi_scratch[kEpiScratch];
  const int tile = blockIdx.x;
  const int row0 = blockIdx.y * kChunkRows;
  const int t = threadIdx.x;
  const int nrows = min(kChunkRows, p.M - row0);
  const WT* const* wseg = reinterpret_cast<const WT* const*>(p.w);
  const XT* x = reinterpret_cast<const XT*>(p.x);
  grid_dep_wait();
  grid_dep_launch();
  // side job: this CTA's share of the next launch's RoPE table
  rope_fill_range(p.epi.fill, ((int)blockIdx.y * (int)gridDim.x + (int)blockIdx.x) * 128 + t,
                  (int)(gridDim.x * gridDim.y) * 128);

  // weight row pointer for tile row r
  auto wrow = [&](int r) -> const WT* {
    if (p.paired) return r < kTileN / 2 ? wseg[0] + (size_t)(tile * (kTileN / 2) + r) * p.K
                                        : wseg[1] + (size_t)(tile * (kTileN / 2) + r - kTileN / 2) * p.K;
    const int s = seg_of_tile(p.epi, tile);
    return wseg[s] + (size_t)((tile - p.epi.seg_tile_begin[s]) * kTileN + r) * p.K;
  };

  float acc[kChunkRows];
#pragma unroll
  for (int j = 0; j < kChunkRows; ++j) acc[j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += kKT) {
    for (int e = t; e < kChunkRows * kKT; e += 128) {
      const int r = e / kKT, c = e % kKT;
      const size_t i = (size_t)(row0 + r) * p.ldx + k0 + c;
      xs[r][c] = r < nrows ? to_f32(x[i]) + (p.x_plane ? to_f32(x[i + p.x_plane]) : 0.f) : 0.f;
    }
    for (int e = t; e < kTileN * kKT; e += 128) {
      const int r = e / kKT, c = e % kKT;
      ws[r][c] = to_f32(wrow(r)[k0 + c]);
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKT; ++kk) {
      const float w = ws[t][kk];
#pragma unroll
      for (int j = 0; j < kChunkRows; ++j) acc[j] = fmaf(xs[j][kk], w, acc[j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < kChunkRows; ++j) chunk[j * kChunkLd + t] = acc[j];
  epilogue_row_scales(p.epi, row0, nrows, epi_scratch, t);
  __syncthreads();
  epilogue_chunk(p.epi, tile, row0, nrows, chunk, t, epi_scratch);
}

cudaError_t launch_gemm_simt(const GemmSimtParams& p, int n_tiles, cudaStream_t st, bool pdl) {
  const dim3 grid((unsigned)n_tiles, (unsigned)((p.M + kChunkRows - 1) / kChunkRows)), block(128);
  if (p.w_bf16 && p.x_bf16) return launch_kernel(gemm_simt_kernel<__nv_bfloat16, __nv_bfloat16>, grid, block, 0, st, pdl, p);
  if (!p.w_bf16 && !p.x_bf16) return launch_kernel(gemm_simt_kernel<float, float>, grid, block, 0, st, pdl, p);
  if (p.w_bf16) return launch_kernel(gemm_simt_kernel<__nv_bfloat16, float>, grid, block, 0, st, pdl, p);
  return launch_kernel(gemm_simt_kernel<float, __nv_bfloat16>, grid, block, 0, st, pdl, p);
}

}  // namespace dfl
