// Internal declarations shared by the host and device translation units of libsage.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "../../include/sage.h"

namespace sage {

constexpr int kSV = 8;          // subvector length v
constexpr int kGroupSV = 16;    // subvectors per radius group (G = 128 weights)
constexpr int kWsHeader = 256;  // bytes reserved for the device status word
constexpr int kBlockOct = 32;   // row octets per storage block (256 rows)

// Device status word bits (first word of the workspace).
constexpr uint32_t kDevTimeout = 1u;
constexpr uint32_t kDevBadInput = 4u;  // an input value found invalid on the device
constexpr uint32_t kDevUnsupported = 2u;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates one matrix descriptor; returns SAGE_OK or the error.
int check_matrix(const sage_matrix* A);

// Per-device facts, looked up with the device current at the time of the call.
constexpr int kMaxDevices = 64;
int current_device();        // -1 when no device can be queried
int current_sm_count();      // SM count of the current device (cached per device)

// Raises a kernel's dynamic shared-memory limit on the current device when a
// launch needs more than any earlier launch on that device did.
class SmemLimit {
  public:
    template <class K>
    bool ensure(K kernel, int bytes) {
        const int dev = current_device();
        if (dev < 0 || dev >= kMaxDevices) return false;
        std::lock_guard<std::mutex> lock(mu_);
        if (bytes <= done_[dev]) return true;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return false;
        done_[dev] = bytes;
        return true;
    }

  private:
    std::mutex mu_;
    int done_[kMaxDevices] = {};
};

// Kernel launchers (sage_gemv.cu / sage_hooks.cu / sage_gemm_sm100.cu).
struct GemvJob {
    sage_matrix A;
    const uint16_t* x;   // [M][d_in] original order (GEMV) or x_perm (GEMM)
    uint16_t* y;         // [M][d_out]
};
int launch_gemv(const GemvJob* jobs, int n, int M, void* ws, size_t ws_bytes, sage_stream_t stream);
size_t gemv_workspace_bytes(const sage_matrix* mats, int n, int M);

int launch_moe(const sage_matrix* experts, int n_experts, const int32_t* pair_expert,
               const int32_t* pair_xrow, int n_pairs, const uint16_t* x, uint16_t* y,
               void* ws, size_t ws_bytes, sage_stream_t stream);
size_t moe_workspace_bytes(const sage_matrix* experts, int n_experts, int n_pairs);
size_t abs_workspace_bytes(int n);  // partials for n candidates scored per synchronisation

int launch_gemm(const sage_matrix* A, const uint16_t* x, int M, uint16_t* y,
                void* ws, size_t ws_bytes, sage_stream_t stream);
size_t gemm_workspace_bytes(const sage_matrix* A, int M);

int launch_dequant(const sage_matrix* A, uint16_t* W, sage_stream_t stream);
int launch_unpack(const sage_matrix* A, uint8_t* signs, uint16_t* idx, uint8_t* q, uint16_t* mu,
                  uint16_t* delta, sage_stream_t stream);
int launch_permute(const uint16_t* x, const int32_t* perm, int M, int d_in, uint16_t* xp,
                   sage_stream_t stream);
int read_and_clear_status(void* ws, sage_stream_t stream);

}  // namespace sage
