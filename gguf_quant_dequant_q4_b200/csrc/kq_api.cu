// C ABI entry points (include/kq.h): host-side argument validation, status
// codes and launch.  No entry point allocates device memory or synchronizes.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "../../include/kq.h"
#include "kq_launch.h"

namespace kq {

namespace {
thread_local int g_last_cuda = 0;
__device__ int g_device_status = 0;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int g_smem_optin[kMaxDevices] = {0};
int* g_status_ptr[kMaxDevices] = {nullptr};

int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d < kMaxDevices ? d : 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_geometry(int type, int* vpb, int* bpb) {
    switch (type) {
    case KQ_Q4_K: *vpb = 256; *bpb = 144; return KQ_OK;
    case KQ_Q6_K: *vpb = 256; *bpb = 210; return KQ_OK;
    case KQ_Q8_0: *vpb = 32; *bpb = 34; return KQ_OK;
    case KQ_Q5_K: *vpb = 256; *bpb = 176; return KQ_OK;
    case KQ_Q4_0: *vpb = 32; *bpb = 18; return KQ_OK;
    default: return KQ_ERR_UNSUPPORTED;
    }
}

// Largest k of any call: the kernels count a row's values and blocks in
// 32-bit integers.
constexpr int64_t kMaxK = (int64_t(1) << 31) - 1;

// Common checks of (codec, W, n, k): codec known, k a positive block multiple
// of at most kMaxK values, n >= 0, W non-null and 16-byte aligned when there
// is work.
int check_weights(int type, const void* w, int64_t n, int64_t k) {
    int vpb, bpb;
    if (block_geometry(type, &vpb, &bpb)) return KQ_ERR_UNSUPPORTED;
    if (k <= 0 || k > kMaxK || k % vpb != 0 || n < 0) return KQ_ERR_INVALID_ARG;
    if (n > 0 && !w) return KQ_ERR_INVALID_ARG;
    if (n > 0 && !aligned16(w)) return KQ_ERR_ALIGNMENT;
    return KQ_OK;
}
}  // namespace

int record_cuda(cudaError_t e) {
    if (e == cudaSuccess) return KQ_OK;
    g_last_cuda = static_cast<int>(e);
    return KQ_ERR_CUDA;
}

int check_launch() { return record_cuda(cudaGetLastError()); }

bool use_pdl() {
    static const bool on = [] {
        const char* v = std::getenv("KQ_NO_PDL");
        return !(v && v[0] == '1');
    }();
    return on;
}

bool use_pair_mma() {
    static const bool on = [] {
        const char* v = std::getenv("KQ_QMM_1SM");
        return !(v && v[0] == '1');
    }();
    return on;
}

int device_sm_count() {
    const int d = current_device();
    if (!g_sm_count[d]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d);
        g_sm_count[d] = v > 0 ? v : 1;
    }
    return g_sm_count[d];
}

int device_smem_optin() {
    const int d = current_device();
    if (!g_smem_optin[d]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d);
        g_smem_optin[d] = v > 0 ? v : 48 * 1024;
    }
    return g_smem_optin[d];
}

int* device_status_ptr() {
    const int d = current_device();
    if (!g_status_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) == cudaSuccess) g_status_ptr[d] = static_cast<int*>(p);
    }
    return g_status_ptr[d];
}

}  // namespace kq

using namespace kq;

extern "C" {

int kq_block_info(int type, int* values_per_block, int* bytes_per_block) {
    int v, b;
    const int rc = block_geometry(type, &v, &b);
    if (rc) return rc;
    if (values_per_block) *values_per_block = v;
    if (bytes_per_block) *bytes_per_block = b;
    return KQ_OK;
}

const char* kq_status_string(int status) {
    switch (status) {
    case KQ_OK: return "ok";
    case KQ_ERR_INVALID_ARG: return "invalid argument";
    case KQ_ERR_UNSUPPORTED: return "unsupported codec or shape";
    case KQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case KQ_ERR_CUDA: return "CUDA runtime error";
    case KQ_ERR_DEVICE_DATA: return "invalid device data";
    default: return "unknown status";
    }
}

int kq_last_cuda_error(void) { return g_last_cuda; }

int kq_read_device_status(int32_t* host_status, int clear) {
    if (!host_status) return KQ_ERR_INVALID_ARG;
    int* p = device_status_ptr();
    if (!p) return KQ_ERR_CUDA;
    // every stream of the device, blocking or not, has finished its kernels
    // before the word is read (a plain copy would order with the legacy
    // default stream only)
    int rc = record_cuda(cudaDeviceSynchronize());
    if (rc) return rc;
    rc = record_cuda(cudaMemcpy(host_status, p, sizeof(int32_t), cudaMemcpyDeviceToHost));
    if (rc) return rc;
    if (clear) {
        const int32_t zero = 0;
        rc = record_cuda(cudaMemcpy(p, &zero, sizeof(int32_t), cudaMemcpyHostToDevice));
    }
    return rc;
}

int kq_set_wait_limit(int64_t ns) { return set_stream_wait_limit(ns > 0 ? static_cast<uint64_t>(ns) : 0); }

int kq_dequantize(int type, const void* w, int64_t n_rows, int64_t k, float* out, void* stream) {
    int rc = check_weights(type, w, n_rows, k);
    if (rc) return rc;
    if (n_rows == 0) return KQ_OK;
    if (!out) return KQ_ERR_INVALID_ARG;
    if (!aligned16(out)) return KQ_ERR_ALIGNMENT;
    return launch_dequantize(type, w, n_rows, k, out, static_cast<cudaStream_t>(stream));
}

int kq_quantize(int type, const float* w, int64_t n_rows, int64_t k, void* out, void* stream) {
    int vpb, bpb;
    if (block_geometry(type, &vpb, &bpb)) return KQ_ERR_UNSUPPORTED;
    if (k <= 0 || k > kMaxK || k % vpb != 0 || n_rows < 0) return KQ_ERR_INVALID_ARG;
    if (n_rows == 0) return KQ_OK;
    if (!w || !out) return KQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(out)) return KQ_ERR_ALIGNMENT;
    return launch_quantize(type, w, n_rows, k, out, static_cast<cudaStream_t>(stream));
}

int kq_qmv(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m, float* y, void* stream) {
    int rc = check_weights(type, w, n, k);
    if (rc) return rc;
    if (m < 1 || m > 16) return KQ_ERR_INVALID_ARG;
    if (n == 0) return KQ_OK;
    if (!x || !y) return KQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return KQ_ERR_ALIGNMENT;
    return launch_qmv(type, w, n, k, x, static_cast<int>(m), y, static_cast<cudaStream_t>(stream));
}

int kq_qmm(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m, float* y, void* stream) {
    int rc = check_weights(type, w, n, k);
    if (rc) return rc;
    if (m < 0 || m > (int64_t(1) << 31) - 1 || n > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID_ARG;
    if (n == 0 || m == 0) return KQ_OK;
    if (!x || !y) return KQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return KQ_ERR_ALIGNMENT;
    return launch_qmm(type, w, n, k, x, m, y, static_cast<cudaStream_t>(stream));
}

int kq_moe_sort(const int32_t* topk_ids, int64_t n_tokens, int32_t top_k, int32_t n_experts, const uint16_t* x,
                int64_t k, uint32_t* sorted_ids, int32_t* sorted_pair, int32_t* inv_order, uint16_t* x_sorted,
                int32_t* err_flag, void* stream) {
    if (n_tokens < 0 || top_k < 1 || n_experts < 1 || n_experts > 256) return KQ_ERR_INVALID_ARG;
    // the token count is bounded first, so that the pair count cannot overflow
    if (n_tokens > (int64_t(1) << 30) || n_tokens * top_k > (int64_t(1) << 30)) return KQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return KQ_OK;
    if (!topk_ids || !sorted_ids || !sorted_pair) return KQ_ERR_INVALID_ARG;
    if (x_sorted) {
        if (!x || k <= 0 || k > kMaxK || k % 8 != 0) return KQ_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(x_sorted)) return KQ_ERR_ALIGNMENT;
    }
    return launch_moe_sort(topk_ids, n_tokens, top_k, n_experts, x, k, sorted_ids, sorted_pair, inv_order, x_sorted,
                           err_flag, static_cast<cudaStream_t>(stream));
}

int kq_expert_tile_map(const uint32_t* sorted_ids, int64_t rows, int32_t n_experts, uint32_t* map, int64_t cap,
                       uint32_t* count, int32_t* err_flag, void* stream) {
    if (rows < 0 || rows > (int64_t(1) << 30) || n_experts < 1 || n_experts > 256) return KQ_ERR_INVALID_ARG;
    if (!map || !count || (rows > 0 && !sorted_ids)) return KQ_ERR_INVALID_ARG;
    if (cap < (rows + 63) / 64 + n_experts) return KQ_ERR_INVALID_ARG;
    return launch_tile_map(sorted_ids, rows, n_experts, map, cap, count, err_flag, static_cast<cudaStream_t>(stream));
}

int kq_gather_qmm(int type, const void* w_bank, int32_t n_experts, int64_t n, int64_t k, const uint16_t* x_sorted,
                  int64_t rows, const uint32_t* map, const uint32_t* count, int64_t cap, float* y, int32_t* err_flag,
                  void* stream) {
    if (n_experts < 1 || n_experts > 256) return KQ_ERR_INVALID_ARG;
    int rc = check_weights(type, w_bank, n, k);
    if (rc) return rc;
    if (rows < 0 || rows > (int64_t(1) << 31) - 1 || cap < 0) return KQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(n_experts) * n > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID_ARG;
    if (n == 0 || rows == 0) return KQ_OK;
    if (!x_sorted || !map || !count || !y) return KQ_ERR_INVALID_ARG;
    if (!aligned16(x_sorted) || !aligned16(y)) return KQ_ERR_ALIGNMENT;
    return launch_gather_qmm(type, w_bank, n_experts, n, k, x_sorted, rows, map, count, cap, y, err_flag,
                             static_cast<cudaStream_t>(stream));
}

int kq_gather_qmv(int type, const void* w_bank, int32_t n_experts, int64_t n, int64_t k, const uint16_t* x,
                  int32_t x_per_token, const int32_t* ids, int64_t n_tokens, int32_t top_k, float* y,
                  int32_t* err_flag, void* stream) {
    if (n_experts < 1 || n_experts > 256 || n_tokens < 0 || top_k < 1) return KQ_ERR_INVALID_ARG;
    int rc = check_weights(type, w_bank, n, k);
    if (rc) return rc;
    if (n_tokens > 8192 || n_tokens * top_k > 8192) return KQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(n_experts) * n > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID_ARG;
    if (n == 0 || n_tokens == 0) return KQ_OK;
    if (!x || !ids || !y) return KQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return KQ_ERR_ALIGNMENT;
    const int pairs = static_cast<int>(n_tokens * top_k);
    // distinct experts per token bound the pairs of one expert by n_tokens
    const int m_cap = n_tokens < 16 ? static_cast<int>(n_tokens) : 16;
    return launch_gather_qmv(type, w_bank, nullptr, 0, 0.f, n_experts, n, k, x, x_per_token ? top_k : 1, ids, pairs,
                             m_cap, y, err_flag, static_cast<cudaStream_t>(stream));
}

int kq_moe_glu_gather(int type, const void* gate_bank, const void* up_bank, int32_t n_experts, int64_t n, int64_t k,
                      const uint16_t* x, const int32_t* ids, int64_t n_tokens, int32_t top_k, int32_t act,
                      float limit, float* out, int32_t* err_flag, void* stream) {
    if (n_experts < 1 || n_experts > 256 || n_tokens < 0 || top_k < 1) return KQ_ERR_INVALID_ARG;
    if (act < KQ_ACT_SILU || act > KQ_ACT_SILU_LIMIT) return KQ_ERR_INVALID_ARG;
    if (act == KQ_ACT_SILU_LIMIT && !(limit > 0.f)) return KQ_ERR_INVALID_ARG;
    int rc = check_weights(type, gate_bank, n, k);
    if (rc) return rc;
    rc = check_weights(type, up_bank, n, k);
    if (rc) return rc;
    if (n_tokens > 8192 || n_tokens * top_k > 8192) return KQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(n_experts) * n > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID_ARG;
    if (n == 0 || n_tokens == 0) return KQ_OK;
    if (!x || !ids || !out) return KQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return KQ_ERR_ALIGNMENT;
    const int pairs = static_cast<int>(n_tokens * top_k);
    const int m_cap = n_tokens < 16 ? static_cast<int>(n_tokens) : 16;
    return launch_gather_qmv(type, gate_bank, up_bank, act, limit, n_experts, n, k, x, top_k, ids, pairs, m_cap, out,
                             err_flag, static_cast<cudaStream_t>(stream));
}

int kq_gather_mix(const float* y, int64_t rows, int64_t n, const int32_t* inv_order, const float* scores,
                  int64_t n_tokens, int32_t top_k, float* out, int32_t* err_flag, void* stream) {
    if (rows < 0 || n < 0 || n % 4 != 0 || n_tokens < 0 || top_k < 1 || top_k > 64) return KQ_ERR_INVALID_ARG;
    if (n_tokens > (int64_t(1) << 31) - 1 || rows > (int64_t(1) << 31) - 1) return KQ_ERR_INVALID_ARG;
    if (n == 0 || n_tokens == 0) return KQ_OK;
    if (!inv_order || !scores || !out || (rows > 0 && !y)) return KQ_ERR_INVALID_ARG;
    if ((y && !aligned16(y)) || !aligned16(out)) return KQ_ERR_ALIGNMENT;
    return launch_gather_mix(y, rows, n, inv_order, scores, n_tokens, top_k, out, err_flag,
                             static_cast<cudaStream_t>(stream));
}

}  // extern "C"
