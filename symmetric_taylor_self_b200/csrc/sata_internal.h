// Internal declarations shared by the libsata translation units.
#pragma once

#include <cstdint>
#include <functional>
#include <vector>

#include <cuda_runtime.h>

#include "sata.h"

namespace sata {

constexpr int kMaxDK = 128;
constexpr int kMaxDV = 128;
constexpr int kMaxP = 8;      // degrees 0..7: a feature is at most seven indices (two packed words)
constexpr int kMaxPStatic = 4;   // the allocation-free decode step derives its basis for P <= 4

// Host copy of the basis (sata_build_basis serves from it).
struct HostBasis {
    int d_K = 0, P = 0;
    std::vector<std::vector<uint8_t>> tuples;  // [F] nondecreasing indices
    std::vector<uint8_t> degree;               // [F]
    std::vector<uint32_t> mult;                // [F] C_p
    std::vector<int64_t> offsets;              // [P+1]
};

int64_t binom64(int n, int k);
int64_t num_features(int d_K, int P);
bool build_basis_host(int d_K, int P, HostBasis &hb);

// Device copy of the basis for the kernels, cached per (device, d_K, P).
//   packed[f] = a | b << 8 | l << 16 | p << 24: the feature's last three indices,
//   where index d_K stands for the constant 1 (tuples of degree < 3 are
//   left-padded with it, so every feature is a "prefix pair (a, b) times a last
//   index l");
//   packed_hi[f] (only when P > 4, else null) = its leading indices i0..i3 of a
//   degree-p tuple, p > 3 (i0 | i1 << 8 | i2 << 16 | i3 << 24, padded with d_K):
//   feature f = x[packed_hi] * x[a] * x[b] * x[l].
//   coef[f]  = alpha_p * C_p[f] = C_p[f] / (p! c^p), c = sqrt(d_K)  (fp32)
//   mcoef[f] = C_p[f] / p! = 1 / prod(mult!)                     (fp32)
struct DeviceBasis {
    int d_K = 0, P = 0;
    int64_t F = 0;
    int64_t offsets[kMaxP + 1] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t *packed = nullptr;
    uint32_t *packed_hi = nullptr;
    float *coef = nullptr;
    float *mcoef = nullptr;
};

// Device-side status words, one set per device: [0] timeout, [1] range.
enum { kFlagTimeout = 0, kFlagRange = 1, kNumFlags = 4 };

// Record a failed CUDA call for sata_last_cuda_error(); returns SATA_ECUDA.
int record_cuda_error(cudaError_t e);

// Library-owned per-device resources (basis cache, status flags, workspaces).
const DeviceBasis *device_basis(int d_K, int P, cudaError_t *err);
int *device_flags(cudaError_t *err);
void *device_workspace(int slot, size_t bytes, cudaError_t *err);
// Immutable device table of `bytes` bytes, built once per (device, key): `fill`
// writes the host image, which is copied to the device.  Freed by sata_shutdown.
const void *device_table(uint64_t key, size_t bytes, const std::function<void(uint8_t *)> &fill,
                         cudaError_t *err);

// Kernel identities for launch statistics.
enum KernelId {
    kDecodeStream = 0, kDecodeFinish, kSimtScan, kSimtFinish, kTcPrep, kTcScan, kTcFinish, kTcReduce,
    kBwdR, kBwdQScan, kBwdKVScan, kBwdFinish, kStateAdd, kBwdTcPrep, kBwdTcScan, kBwdTcFinish, kTcStats,
    kTcStateStats, kBwdTcR, kNumKernels
};
const char *kernel_name(int id);
// Call around every kernel launch: begin() records a start event when timing is
// on, end() records the stop event and counts the launch.
void launch_begin(int id, cudaStream_t s);
void launch_end(int id, cudaStream_t s);

// Runtime options.
extern int64_t g_opt_prefill_path;
extern int64_t g_opt_wait_limit;
extern int64_t g_opt_test_stall;
extern int64_t g_opt_time_kernels;
extern int64_t g_opt_deterministic;

// ---- decode (decode.cu) ----
size_t decode_workspace_bytes(int BH, int64_t F, int d_V);
cudaError_t launch_decode(const DeviceBasis &basis, int BH, int d_V, float *S, float *Z,
                          const void *q, const void *k, const void *v, float *out,
                          float *partials, cudaStream_t stream);

// ---- prefill, CUDA-core path (prefill_simt.cu) ----
size_t prefill_simt_workspace_bytes(int BH, int64_t N, int64_t F, int d_V, bool need_state);
cudaError_t launch_prefill_simt(const DeviceBasis &basis, int BH, int64_t N, int d_V,
                                const void *q, const void *k, const void *v, float *out,
                                float *S, float *Z, bool state_in, void *ws, size_t ws_bytes,
                                cudaStream_t stream, float *den_out = nullptr, bool f32_in = false);

// ---- state operations (state_ops.cu) ----
// S += dS (nS floats), Z += dZ (nZ floats), on `stream`.
cudaError_t launch_state_add(float *S, float *Z, const float *dS, const float *dZ, int64_t nS, int64_t nZ,
                             cudaStream_t stream);

// ---- backward of the prefill on tensor cores (backward_tc.cuh via prefill_tc.cu) ----
// Shapes of the tensor-core prefill; the gradient scans add into their sums with atomics.
bool prefill_backward_tc_supported(int d_K, int d_V, int P);
size_t prefill_backward_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P);
cudaError_t launch_prefill_backward_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V, const void *q,
                                       const void *k, const void *v, const float *dy, float *dq, float *dk,
                                       float *dv, void *ws, size_t ws_bytes, int *flags, cudaStream_t stream);

// ---- backward of the prefill, CUDA-core path (backward_simt.cu) ----
size_t prefill_backward_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool use_tc);
// The forward it recomputes runs on tensor cores when use_tc (flags: the device status words).
cudaError_t launch_prefill_backward(const DeviceBasis &basis, int BH, int64_t N, int d_V,
                                    const void *q, const void *k, const void *v, const float *dy,
                                    float *dq, float *dk, float *dv, void *ws, size_t ws_bytes,
                                    bool use_tc, int *flags, cudaStream_t stream);

// ---- prefill, tensor-core path (prefill_tc.cu) ----
// Host-buffer prefill: the kernels read and write the device copies passed as q, k, v, out;
// each token segment's inputs are copied in on h2d, and its output copied back on d2h,
// so transfers overlap the other segments' compute.
struct HostIO {
    const void *q, *k, *v;   // host [BH][N][d] bf16
    float *out;              // host [BH][N][d_V] fp32
    cudaStream_t h2d, d2h;   // copy streams
    cudaStream_t aux;        // a segment's prep and finish, beside the scans
};
constexpr int kHostSegments = 4;   // at least this many segments when copies are pipelined
bool prefill_tc_supported(int d_K, int d_V, int P);
size_t prefill_tc_workspace_bytes(int BH, int64_t N, int64_t F, int d_K, int d_V, int P, bool need_state,
                                  bool host_io);
cudaError_t launch_prefill_tc(const DeviceBasis &basis, int BH, int64_t N, int d_V,
                              const void *q, const void *k, const void *v, float *out,
                              float *S, float *Z, bool state_in, void *ws, size_t ws_bytes,
                              int *flags, cudaStream_t stream, const HostIO *io, float *den_out = nullptr);
// Library-owned copy streams of the current device (non-blocking), created once.
cudaError_t device_copy_streams(cudaStream_t *h2d, cudaStream_t *d2h, cudaStream_t *aux);

}  // namespace sata
