// Private definition of mk_handle, shared by the C-ABI translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <vector>

#include "mk.h"
#include "runtime.cuh"
#include "tgraph.hpp"

namespace mk {
size_t worker_smem_bytes(int stages, int stage_bytes, int pps, int head_dim, int rep_p);
cudaError_t worker_configure(size_t smem);
cudaError_t worker_max_blocks(int *blocks, size_t smem);
cudaError_t launch_persistent(const Params &p, int workers, size_t smem, cudaStream_t stream);
cudaError_t launch_tasks(const Params &p, int n_ctas, size_t smem, cudaStream_t stream);
cudaError_t permute_to_fragments(void *dst, const void *src, int rows, int K,
                                 cudaStream_t stream);
}  // namespace mk

struct mk_handle;
namespace mk {
// Encodes p->tmap_k / p->tmap_v for the caches of one step; returns "" or
// the reason it failed.
std::string encode_kv_maps(const mk_handle *h, const void *k_cache, const void *v_cache,
                           Params *p);
}  // namespace mk

struct mk_handle {
  mk_model_config cfg{};
  mk_tuning tune{};
  mk::TaskGraph graph;
  bool host_only = true;
  int device = -1;
  std::string err;
  // device state
  void *dev_block = nullptr;  // graph tables, counters, activations, rope table
  size_t dev_block_bytes = 0;
  void *arena = nullptr;      // weights
  size_t arena_bytes = 0;
  bool loaded = false;
  mk::DevLayer *d_layers = nullptr;
  std::vector<mk::DevLayer> layers;
  std::vector<int32_t> op_offset;  // into d_op_tasks
  int32_t *d_op_tasks = nullptr;
  mk::Params base{};
  size_t smem = 0;
  int64_t act_bytes = 0;
  int64_t weight_bytes = 0;
};


