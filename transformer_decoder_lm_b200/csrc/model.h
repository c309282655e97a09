// model.h - the handle behind gpt2_handle_t and the helpers the C ABI files
// share (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "gpt2.h"
#include "kernels.h"

namespace g2 {

// Weight tensor maps are kept for every box height a GEMM pick can ask for:
// the tile widths (single CTA) and their halves (CTA pairs: 96 for 192).
constexpr int NUM_BOX = 5;
constexpr int BOX_ROWS[NUM_BOX] = {256, 192, 128, 96, 64};
inline int box_index(int rows) {
  return rows == 256 ? 0 : (rows == 192 ? 1 : (rows == 128 ? 2 : (rows == 96 ? 3 : 4)));
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct LayerPtrs {
  const void *ln1_g, *ln1_b, *attn_w, *attn_b, *attn_proj_w, *attn_proj_b;
  const void *ln2_g, *ln2_b, *fc_w, *fc_b, *mlp_proj_w, *mlp_proj_b;
};

struct WeightMaps {  // one tensor map per box height
  CUtensorMap attn[NUM_BOX], proj[NUM_BOX], fc[NUM_BOX], mproj[NUM_BOX];
};

// Byte offsets of the workspace slices (gpt2_create).
struct Plan {
  size_t x, h, qkv, y, f, part, tgt, tok, attn, attn_flags, status, total;
  int attn_pairs;
};

}  // namespace g2

struct gpt2_model {
  gpt2_config_t cfg;
  bool bf16;
  int device = 0, num_sms = 0;
  int max_B = 0, max_T = 0;
  long max_M = 0;
  const void *wte = nullptr, *wpe = nullptr, *lnf_g = nullptr, *lnf_b = nullptr;
  std::vector<g2::LayerPtrs> layers;
  std::vector<g2::WeightMaps> maps;
  CUtensorMap wte_map[g2::NUM_BOX];
  uint8_t* ws = nullptr;
  g2::Plan plan;
  float* x = nullptr;
  void *h = nullptr, *qkv = nullptr, *y = nullptr, *f = nullptr;
  float2* part = nullptr;
  float* tgt = nullptr;
  float* tok = nullptr;
  int* status = nullptr;
  g2::AttnScratch attn;        // attention work counters (in the zeroed status block), split flags, partials
  uint64_t launches = 0;
  cudaEvent_t ev_lm_begin = nullptr, ev_lm_end = nullptr;
};
