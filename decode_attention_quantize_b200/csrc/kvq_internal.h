// Kernel parameter blocks and launchers shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <utility>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

struct AppendParams {
  int B, H, n_new;
  int k_scheme, v_scheme;
  int in_bf16;
  int paged, cap, page_size, max_pages, num_pages;
  int pos0;  // dense: first position written (quantized tokens so far)
  int rcap;
  const void* k_new;
  const void* v_new;
  const int32_t* new_lens;
  void* k_codes;
  void* v_codes;
  float* k_scale;
  float* k_zero;
  float* v_scale;
  float* v_zero;
  uint8_t* k_zp;
  uint8_t* v_zp;
  uint16_t* k_res;
  uint16_t* v_res;
  const int32_t* page_table;
  int32_t* seq_lens;
  uint32_t* status;
  int rotate;  // rows rotated by the normalised Walsh-Hadamard transform before quantization
  int group;   // INT4 per-group: channels per group (32, 64 or 128)
};

struct DequantParams {
  int B, H, T_out, which, scheme;
  int paged, cap, page_size, max_pages, num_pages;
  int len_q, len_res, rcap;
  const uint8_t* codes;
  const float* scale;
  const float* zero;
  const uint8_t* zp;
  const uint16_t* res;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint32_t* status;
  float* out;
  int rotate;  // rotate each dequantized row back
  int group;   // INT4 per-group: channels per group
};

struct DecodeParams {
  int B, Hq, Hkv, G, HG;        // G = Hq / Hkv, HG = ceil(G / 8) head groups of 8
  int k_scheme, v_scheme;
  int paged, cap, page_size, max_pages, num_pages;
  int len_q, len_res, rcap;     // dense lengths (uniform over the batch)
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const float* k_scale;
  const float* k_zero;
  const float* v_scale;
  const float* v_zero;
  const uint8_t* k_zp;
  const uint8_t* v_zp;
  const uint16_t* k_res;
  const uint16_t* v_res;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint32_t* status;
  const void* q;
  int q_bf16;
  float softmax_scale;
  float* out;
  float* lse;
  // workspace
  float* part_o;                // [slots, 8, 128]
  float* part_ml;               // [slots, 8, 2]
  int32_t* plan;                // paged: [2B + 2] tile prefix over sequences, then lengths
  int ncta;
  int n_pairs;
  int ts;                       // tokens per quantized tile of the chosen kernel
  int nq, nr;                   // dense: quantized / residual tiles per pair
  int rotate;                   // rotate each query, and each output back
  int group;                    // INT4 per-group: channels per group (selects the kernel)
  float rope_theta;             // > 0: keys cached before RoPE, rotated at their positions here
  // >= 0: the kernel runs as the programmatic dependent of an append that writes token
  // positions from here on (and nothing else the decode reads): tiles before it are read
  // before the wait for that append, the others after it. < 0: wait at the start.
  int early_from;
};

constexpr int kMaxCtas = 1024;

// Count of kernel launches issued by the library (reported by kvq_launch_count).
void count_launches(int n);  // decode grid bound used to size the workspace

// Append modes: plain (the scales in the cache), calibrating (scales from the block), or
// rescaling (the block's scales merged into the cached ones, cached codes requantized).
enum { kAppendPlain = 0, kAppendCalibrate = 1, kAppendRescale = 2 };
// Workspace: calibration keys, then (rescaling) the offset below: old scales [2][H*128]
// fp32, old zero points [2][H*128] uint8, two changed flags.
size_t rescale_ws_offset(int H);
cudaError_t launch_append(const AppendParams& p, void* workspace, int mode, int r_old, int flushed, int r_new,
                          cudaStream_t st);
cudaError_t launch_dequantize(const DequantParams& p, cudaStream_t st);
// Launch with programmatic dependent launch: the kernel may be scheduled while the previous
// kernel in the stream is still running and must call griddepcontrol.wait before it touches
// memory that kernel writes (or reads, for memory it overwrites).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Returns cudaErrorNotSupported when the (k_scheme, v_scheme, layout) pair has no kernel.
cudaError_t launch_decode(DecodeParams p, cudaStream_t st);
bool decode_supported(int k_scheme, int v_scheme, int paged, int group, bool rope);
bool append_pair_supported(int k_scheme, int v_scheme);
// Streaming multiprocessors of the current device (cached per device).
int sm_count();

}  // namespace kvq
