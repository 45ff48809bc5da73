// Host-side declarations shared by the kq translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kq.h"

namespace kq {

// Number of SMs of the current device (cached per device).
int device_sm_count();
// Maximum opt-in dynamic shared memory per block of the current device.
int device_smem_optin();
// Records the launch error (if any) and maps it to a kq_status.
int check_launch();
int record_cuda(cudaError_t e);
// Whether kernels are launched with programmatic dependent launch (PDL):
// on unless the environment sets KQ_NO_PDL=1 (an A/B lever).
bool use_pdl();
// Whether the prefill GEMM runs on CTA pairs (tcgen05 cta_group::2, 256
// weight rows per tile): on unless the environment sets KQ_QMM_1SM=1.
bool use_pair_mma();
// Device address of the library-wide status word (bits KQ_DEV_*).
int* device_status_ptr();

int launch_quantize(int type, const float* x, int64_t n_rows, int64_t k, void* out, cudaStream_t s);
int launch_dequantize(int type, const void* w, int64_t n_rows, int64_t k, float* out, cudaStream_t s);
int launch_qmv(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
               cudaStream_t s);
// Staged decode kernel for few activation rows; KQ_ERR_UNSUPPORTED for shapes
// it does not cover.
int launch_qmv_stream(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
                      cudaStream_t s);
// Decode MoE product (one output row per (token, slot) pair) on the staged
// kernel; with w_bank2 (the up bank) the GLU act(x W^T) * (x W2^T) of each
// pair.  KQ_ERR_UNSUPPORTED for shapes it does not cover.
int launch_gather_qmv(int type, const void* w_bank, const void* w_bank2, int act, float limit, int n_experts,
                      int64_t n, int64_t k, const uint16_t* x, int xdiv, const int32_t* ids, int pairs, int m_cap,
                      float* y, int32_t* err_flag, cudaStream_t s);
// Pipeline wait limit (ns; 0 = the default) of the staged decode kernel on
// the current device.
int set_stream_wait_limit(uint64_t ns);
// q5_K / q4_0 decode product: exact fp32 decode and fp32 dot (k % 256 == 0).
int launch_qmv_exact(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
                     cudaStream_t s);
int launch_qmm(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m, float* y,
               cudaStream_t s);
int launch_gather_qmm(int type, const void* w_bank, int n_experts, int64_t n, int64_t k,
                      const uint16_t* x_sorted, int64_t rows, const uint32_t* map, const uint32_t* count,
                      int64_t cap, float* y, int32_t* err_flag, cudaStream_t s);
int launch_moe_sort(const int32_t* topk_ids, int64_t n_tokens, int top_k, int n_experts, const uint16_t* x,
                    int64_t k, uint32_t* sorted_ids, int32_t* sorted_pair, int32_t* inv_order,
                    uint16_t* x_sorted, int32_t* err_flag, cudaStream_t s);
int launch_gather_mix(const float* y, int64_t rows, int64_t n, const int32_t* inv_order, const float* scores,
                      int64_t n_tokens, int top_k, float* out, int32_t* err_flag, cudaStream_t s);
int launch_tile_map(const uint32_t* sorted_ids, int64_t rows, int n_experts, uint32_t* map, int64_t cap,
                    uint32_t* count, int32_t* err_flag, cudaStream_t s);

}  // namespace kq
