// Dynamic block-size scheduling ("DFlash – 플래시 추측적 디코딩을 위한 블록 확산" §3
// item 4, §4: the drafter trained at block 16 also runs with smaller blocks, the
// block size being scheduled dynamically).
//
// Device side: the per-position acceptance counts of a cycle's verify results,
// accumulated with integer atomics (order-independent, exact). A cycle run with
// block B whose request accepted a drafts tested positions 1 .. min(a+1, B-1)
// and accepted positions 1 .. a.
//
// Host side: the policy keeps decayed counts T_i, A_i, estimates
// alpha_i = (A_i + 1) / (T_i + 2) (a Beta(1, 1) prior), the expected tokens of a
// cycle with block B as 1 + sum_{i<B} prod_{j<=i} alpha_j, and picks the
// candidate block with the most expected tokens per unit of the caller's cycle
// cost (the smaller block on an exact tie).
#include <algorithm>
#include <cmath>
#include <new>
#include <vector>

#include "../../include/dflash.h"
#include "common.cuh"

namespace dfl {

// counts[0 .. n_pos): tested per position, counts[n_pos .. 2 n_pos): accepted per position.
__global__ void acceptance_count_kernel(const int* accepted, int bs, int B, int n_pos, unsigned long long* counts) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= bs * (B - 1)) return;
  const int r = idx / (B - 1), i = idx % (B - 1) + 1;   // position 1 .. B-1
  if (i >= n_pos) return;
  const int a = accepted[r];
  if (i <= a + 1) atomicAdd(counts + i, 1ull);
  if (i <= a) atomicAdd(counts + n_pos + i, 1ull);
}

}  // namespace dfl

extern "C" dflash_status dflash_acceptance_count(const int* d_accepted, int bs, int B, unsigned long long* d_counts,
                                                 int n_pos, void* stream) {
  if (!d_accepted || !d_counts || bs <= 0 || B <= 0 || n_pos <= 0) return DFLASH_ERR_ARG;
  if (B > n_pos) return DFLASH_ERR_ARG;
  if (B == 1) return DFLASH_OK;   // nothing drafted, nothing tested
  const int n = bs * (B - 1);
  dfl::acceptance_count_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      d_accepted, bs, B, n_pos, d_counts);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

struct dflash_block_policy {
  std::vector<int> candidates;   // ascending
  double decay = 1.0;
  std::vector<double> tested, accepted;
};

extern "C" dflash_status dflash_block_policy_create(const int* candidates, int n_candidates, double decay, int n_pos,
                                                    dflash_block_policy** out) {
  if (!out) return DFLASH_ERR_ARG;
  *out = nullptr;
  if (!candidates || n_candidates <= 0 || n_pos <= 0 || !(decay > 0.0 && decay <= 1.0)) return DFLASH_ERR_ARG;
  dflash_block_policy* p = new (std::nothrow) dflash_block_policy();
  if (!p) return DFLASH_ERR_OOM;
  try {
    p->candidates.assign(candidates, candidates + n_candidates);
    std::sort(p->candidates.begin(), p->candidates.end());
    if (p->candidates.front() < 1 || p->candidates.back() > n_pos) {
      delete p;
      return DFLASH_ERR_ARG;
    }
    p->decay = decay;
    p->tested.assign((size_t)n_pos, 0.0);
    p->accepted.assign((size_t)n_pos, 0.0);
  } catch (...) {   // no C++ exception crosses the C ABI
    delete p;
    return DFLASH_ERR_OOM;
  }
  *out = p;
  return DFLASH_OK;
}

extern "C" void dflash_block_policy_destroy(dflash_block_policy* p) { delete p; }

extern "C" dflash_status dflash_block_policy_observe(dflash_block_policy* p, const unsigned long long* tested,
                                                     const unsigned long long* accepted, int n_pos) {
  if (!p || !tested || !accepted || n_pos != (int)p->tested.size()) return DFLASH_ERR_ARG;
  for (int i = 0; i < n_pos; ++i) {
    p->tested[i] = p->decay * p->tested[i] + (double)tested[i];
    p->accepted[i] = p->decay * p->accepted[i] + (double)accepted[i];
  }
  return DFLASH_OK;
}

extern "C" double dflash_block_policy_expected_tokens(const dflash_block_policy* p, int B) {
  if (!p || B < 1 || B > (int)p->tested.size()) return -1.0;
  double total = 1.0, run = 1.0;
  for (int i = 1; i < B; ++i) {
    run *= (p->accepted[i] + 1.0) / (p->tested[i] + 2.0);
    total += run;
  }
  return total;
}

extern "C" int dflash_block_policy_choose(const dflash_block_policy* p, const double* costs, int n_costs) {
  if (!p || !costs || n_costs != (int)p->candidates.size()) return -(int)DFLASH_ERR_ARG;
  int best = p->candidates[0];
  double best_v = -1.0;
  for (int k = 0; k < n_costs; ++k) {
    if (!(costs[k] > 0.0)) return -(int)DFLASH_ERR_ARG;
    const double v = dflash_block_policy_expected_tokens(p, p->candidates[k]) / costs[k];
    if (v > best_v) {
      best = p->candidates[k];
      best_v = v;
    }
  }
  return best;
}

extern "C" int dflash_block_policy_choose_linear(const dflash_block_policy* p, int bs, double c0, double c1) {
  if (!p || bs <= 0 || !(c0 >= 0.0) || !(c1 >= 0.0)) return -(int)DFLASH_ERR_ARG;
  try {
    std::vector<double> costs;
    for (int B : p->candidates) costs.push_back(c0 + c1 * (double)bs * (double)B);
    return dflash_block_policy_choose(p, costs.data(), (int)costs.size());
  } catch (...) {   // no C++ exception crosses the C ABI
    return -(int)DFLASH_ERR_OOM;
  }
}
