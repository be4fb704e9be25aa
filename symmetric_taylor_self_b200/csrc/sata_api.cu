// C ABI of libsata: argument checks, per-device caches, dispatch.
// Every function here is host code; the arithmetic lives in the kernels.
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include <cuda_runtime.h>

#include "sata_internal.h"

namespace sata {

int64_t g_opt_prefill_path = 0;
int64_t g_opt_wait_limit = 0;
int64_t g_opt_test_stall = 0;
int64_t g_opt_deterministic = 0;

namespace {

std::mutex g_mu;
thread_local int g_last_cuda = 0;
cudaStream_t g_stream = nullptr;

struct DeviceRes {
    std::map<std::pair<int, int>, DeviceBasis> bases;
    int *flags = nullptr;
    void *ws[4] = {nullptr, nullptr, nullptr, nullptr};
    size_t ws_bytes[4] = {0, 0, 0, 0};
    std::map<uint64_t, void *> tables;
    cudaStream_t h2d = nullptr, d2h = nullptr, aux = nullptr;
};
std::map<int, DeviceRes> g_dev;
std::map<std::pair<int, int>, HostBasis> g_host_bases;

int cuda_fail(cudaError_t e) {
    g_last_cuda = (int)e;
    return SATA_ECUDA;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool pow2_dv(int d_V) {
    return d_V == 4 || d_V == 8 || d_V == 16 || d_V == 32 || d_V == 64 || d_V == 128;
}

int check_shape(int d_K, int d_V, int P) {
    if (d_K < 1 || d_V < 1 || P < 1) return SATA_EINVAL;
    if (d_K > kMaxDK || d_V > kMaxDV || P > kMaxP || !pow2_dv(d_V)) return SATA_EUNSUPPORTED;
    return SATA_OK;
}

int check_heads(int B, int H, int *BH) {
    if (B < 0 || H < 0) return SATA_EINVAL;
    const int64_t bh = (int64_t)B * H;
    if (bh > INT_MAX) return SATA_EUNSUPPORTED;
    *BH = (int)bh;
    return SATA_OK;
}

const HostBasis *host_basis(int d_K, int P) {
    auto key = std::make_pair(d_K, P);
    auto it = g_host_bases.find(key);
    if (it != g_host_bases.end()) return &it->second;
    HostBasis hb;
    if (!build_basis_host(d_K, P, hb)) return nullptr;
    return &g_host_bases.emplace(key, std::move(hb)).first->second;
}

int current_device(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    return dev;
}

}  // namespace

int record_cuda_error(cudaError_t e) { return cuda_fail(e); }

const DeviceBasis *device_basis(int d_K, int P, cudaError_t *err) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int dev = current_device(err);
    if (*err != cudaSuccess) return nullptr;
    DeviceRes &r = g_dev[dev];
    auto key = std::make_pair(d_K, P);
    auto it = r.bases.find(key);
    if (it != r.bases.end()) return &it->second;
    const HostBasis *hb = host_basis(d_K, P);
    if (!hb) {
        *err = cudaErrorInvalidValue;
        return nullptr;
    }
    const int64_t F = hb->offsets[P];
    std::vector<uint32_t> packed(F), packed_hi(P > 4 ? F : 0);
    std::vector<float> coef(F), mcoef(F);
    const double c = std::sqrt((double)d_K);
    for (int64_t f = 0; f < F; ++f) {
        const auto &t = hb->tuples[f];
        const int p = (int)t.size();
        // last three indices, left-padded with d_K (read as the constant 1)
        uint32_t idx[3] = {(uint32_t)d_K, (uint32_t)d_K, (uint32_t)d_K};
        const int lo = p > 3 ? p - 3 : 0;
        for (int m = lo; m < p; ++m) idx[3 - (p - m)] = t[m];
        packed[f] = idx[0] | (idx[1] << 8) | (idx[2] << 16) | ((uint32_t)p << 24);
        if (P > 4) {   // leading indices of a degree > 3 tuple
            uint32_t hi[4] = {(uint32_t)d_K, (uint32_t)d_K, (uint32_t)d_K, (uint32_t)d_K};
            for (int m = 0; m < lo; ++m) hi[m] = t[m];
            packed_hi[f] = hi[0] | (hi[1] << 8) | (hi[2] << 16) | (hi[3] << 24);
        }
        double pf = 1.0;
        for (int i = 2; i <= p; ++i) pf *= i;
        mcoef[f] = (float)((double)hb->mult[f] / pf);
        coef[f] = (float)((double)hb->mult[f] / (pf * std::pow(c, (double)p)));
    }
    DeviceBasis db;
    db.d_K = d_K;
    db.P = P;
    db.F = F;
    for (int p = 0; p <= P; ++p) db.offsets[p] = hb->offsets[p];
    *err = cudaMalloc(&db.packed, F * sizeof(uint32_t));
    if (*err == cudaSuccess && P > 4) *err = cudaMalloc(&db.packed_hi, F * sizeof(uint32_t));
    if (*err == cudaSuccess && P > 4)
        *err = cudaMemcpy(db.packed_hi, packed_hi.data(), F * sizeof(uint32_t), cudaMemcpyHostToDevice);
    if (*err == cudaSuccess) *err = cudaMalloc(&db.coef, F * sizeof(float));
    if (*err == cudaSuccess) *err = cudaMalloc(&db.mcoef, F * sizeof(float));
    if (*err == cudaSuccess)
        *err = cudaMemcpy(db.packed, packed.data(), F * sizeof(uint32_t), cudaMemcpyHostToDevice);
    if (*err == cudaSuccess)
        *err = cudaMemcpy(db.coef, coef.data(), F * sizeof(float), cudaMemcpyHostToDevice);
    if (*err == cudaSuccess)
        *err = cudaMemcpy(db.mcoef, mcoef.data(), F * sizeof(float), cudaMemcpyHostToDevice);
    if (*err != cudaSuccess) {
        cudaFree(db.packed);
        cudaFree(db.packed_hi);
        cudaFree(db.coef);
        cudaFree(db.mcoef);
        return nullptr;
    }
    return &r.bases.emplace(key, db).first->second;
}

int *device_flags(cudaError_t *err) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int dev = current_device(err);
    if (*err != cudaSuccess) return nullptr;
    DeviceRes &r = g_dev[dev];
    if (!r.flags) {
        *err = cudaMalloc(&r.flags, kNumFlags * sizeof(int));
        if (*err == cudaSuccess) *err = cudaMemset(r.flags, 0, kNumFlags * sizeof(int));
        if (*err != cudaSuccess) {
            cudaFree(r.flags);
            r.flags = nullptr;
        }
    }
    return r.flags;
}

void *device_workspace(int slot, size_t bytes, cudaError_t *err) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int dev = current_device(err);
    if (*err != cudaSuccess) return nullptr;
    DeviceRes &r = g_dev[dev];
    if (r.ws_bytes[slot] < bytes) {
        if (r.ws[slot]) {
            // the old buffer may still be read by enqueued work
            *err = cudaDeviceSynchronize();
            if (*err != cudaSuccess) return nullptr;
            cudaFree(r.ws[slot]);
            r.ws[slot] = nullptr;
            r.ws_bytes[slot] = 0;
        }
        *err = cudaMalloc(&r.ws[slot], bytes);
        if (*err != cudaSuccess) {
            r.ws[slot] = nullptr;
            return nullptr;
        }
        r.ws_bytes[slot] = bytes;
    }
    return r.ws[slot];
}

cudaError_t device_copy_streams(cudaStream_t *h2d, cudaStream_t *d2h, cudaStream_t *aux) {
    std::lock_guard<std::mutex> lk(g_mu);
    cudaError_t err = cudaSuccess;
    const int dev = current_device(&err);
    if (err != cudaSuccess) return err;
    DeviceRes &r = g_dev[dev];
    if (!r.h2d && (err = cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking)) != cudaSuccess) return err;
    if (!r.d2h && (err = cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking)) != cudaSuccess) return err;
    if (!r.aux && (err = cudaStreamCreateWithFlags(&r.aux, cudaStreamNonBlocking)) != cudaSuccess) return err;
    *h2d = r.h2d;
    *d2h = r.d2h;
    *aux = r.aux;
    return cudaSuccess;
}

const void *device_table(uint64_t key, size_t bytes, const std::function<void(uint8_t *)> &fill,
                         cudaError_t *err) {
    std::lock_guard<std::mutex> lk(g_mu);
    const int dev = current_device(err);
    if (*err != cudaSuccess) return nullptr;
    DeviceRes &r = g_dev[dev];
    auto it = r.tables.find(key);
    if (it != r.tables.end()) return it->second;
    std::vector<uint8_t> host(bytes, 0);
    fill(host.data());
    void *d = nullptr;
    *err = cudaMalloc(&d, bytes);
    if (*err == cudaSuccess) *err = cudaMemcpy(d, host.data(), bytes, cudaMemcpyHostToDevice);
    if (*err != cudaSuccess) {
        cudaFree(d);
        return nullptr;
    }
    r.tables[key] = d;
    return d;
}

namespace {

size_t prefill_ws_bytes(int BH, int64_t N, int d_K, int d_V, int P, bool need_state, bool *use_tc,
                        bool host_io = false) {
    const int64_t F = num_features(d_K, P);
    bool tc = false;
    if (g_opt_prefill_path == 2) tc = true;
    else if (g_opt_prefill_path == 0) tc = prefill_tc_supported(d_K, d_V, P);
    if (use_tc) *use_tc = tc;
    return tc ? prefill_tc_workspace_bytes(BH, N, F, d_K, d_V, P, need_state, host_io)
              : prefill_simt_workspace_bytes(BH, N, F, d_V, need_state);
}

// Shared argument checks of the prefill entry points (pointers excepted).
int check_prefill_args(int B, int H, int64_t N, int d_K, int d_V, int P, const sata_state *st, int *BH) {
    int rc = check_heads(B, H, BH);
    if (rc) return rc;
    if (N < 0) return SATA_EINVAL;
    rc = check_shape(d_K, d_V, P);
    if (rc) return rc;
    if (st) {
        if (st->B != B || st->H != H || st->d_K != d_K || st->d_V != d_V || st->P != P)
            return SATA_EINVAL;
        if (!st->S || !st->Z) return SATA_EINVAL;
        if (!aligned16(st->S) || !aligned16(st->Z)) return SATA_EALIGN;
    }
    if (g_opt_prefill_path == 2 && !prefill_tc_supported(d_K, d_V, P)) return SATA_EUNSUPPORTED;
    return SATA_OK;
}

}  // namespace
}  // namespace sata

using namespace sata;

extern "C" {

const char *sata_status_string(int status) {
    switch (status) {
        case SATA_OK: return "SATA_OK";
        case SATA_EINVAL: return "SATA_EINVAL: invalid argument";
        case SATA_EUNSUPPORTED: return "SATA_EUNSUPPORTED: shape outside the supported set";
        case SATA_ECUDA: return "SATA_ECUDA: CUDA runtime or launch error";
        case SATA_ETIMEOUT: return "SATA_ETIMEOUT: a bounded device-side wait expired";
        case SATA_ENOMEM: return "SATA_ENOMEM: workspace allocation failed or too small";
        case SATA_ERANGE: return "SATA_ERANGE: a non-finite input or output in the tensor-core prefill";
        case SATA_EALIGN: return "SATA_EALIGN: device pointer not 16-byte aligned";
        default: return "unknown sata status";
    }
}

int sata_last_cuda_error(void) { return g_last_cuda; }

int sata_version(void) { return 10000; }

int sata_num_features(int d_K, int P, int64_t *F_out) {
    if (d_K < 1 || P < 1 || !F_out) return SATA_EINVAL;
    if (d_K > 255 || P > 8) return SATA_EUNSUPPORTED;
    *F_out = num_features(d_K, P);
    return SATA_OK;
}

int sata_build_basis(int d_K, int P, uint8_t *M, uint32_t *C, int64_t *offsets, int64_t *F_out) {
    if (d_K < 1 || P < 1) return SATA_EINVAL;
    if (d_K > 255 || P > 8) return SATA_EUNSUPPORTED;
    const HostBasis *hb;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        hb = host_basis(d_K, P);
    }
    if (!hb) return SATA_EUNSUPPORTED;
    const int64_t F = hb->offsets[P];
    const int width = P - 1 > 0 ? P - 1 : 1;
    if (M) {
        for (int64_t f = 0; f < F; ++f) {
            const auto &t = hb->tuples[f];
            for (int m = 0; m < width; ++m) M[f * width + m] = m < (int)t.size() ? t[m] : 0xFF;
        }
    }
    if (C) std::memcpy(C, hb->mult.data(), F * sizeof(uint32_t));
    if (offsets) std::memcpy(offsets, hb->offsets.data(), (P + 1) * sizeof(int64_t));
    if (F_out) *F_out = F;
    return SATA_OK;
}

int sata_set_stream(void *stream) {
    g_stream = (cudaStream_t)stream;
    return SATA_OK;
}

int sata_sync_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    int *flags = device_flags(&e);
    if (!flags) return cuda_fail(e);
    int h[kNumFlags];
    e = cudaMemcpy(h, flags, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    int st = SATA_OK;
    if (h[kFlagTimeout]) st = SATA_ETIMEOUT;
    else if (h[kFlagRange]) st = SATA_ERANGE;
    if (st != SATA_OK) {
        e = cudaMemset(flags, 0, sizeof(h));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return st;
}

void sata_shutdown(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto &kv : g_dev) {
        if (cudaSetDevice(kv.first) != cudaSuccess) continue;
        cudaDeviceSynchronize();
        for (auto &b : kv.second.bases) {
            cudaFree(b.second.packed);
            cudaFree(b.second.packed_hi);
            cudaFree(b.second.coef);
            cudaFree(b.second.mcoef);
        }
        cudaFree(kv.second.flags);
        for (int s = 0; s < 4; ++s) cudaFree(kv.second.ws[s]);
        for (auto &t : kv.second.tables) cudaFree(t.second);
        if (kv.second.h2d) cudaStreamDestroy(kv.second.h2d);
        if (kv.second.d2h) cudaStreamDestroy(kv.second.d2h);
        if (kv.second.aux) cudaStreamDestroy(kv.second.aux);
    }
    g_dev.clear();
    cudaSetDevice(cur);
}

int sata_state_bytes(int B, int H, int d_K, int d_V, int P, size_t *S_bytes, size_t *Z_bytes) {
    int BH = 0;
    int rc = check_heads(B, H, &BH);
    if (rc) return rc;
    rc = check_shape(d_K, d_V, P);
    if (rc) return rc;
    const int64_t F = num_features(d_K, P);
    if (S_bytes) *S_bytes = (size_t)BH * F * d_V * sizeof(float);
    if (Z_bytes) *Z_bytes = (size_t)BH * F * sizeof(float);
    return SATA_OK;
}

int sata_state_init(sata_state *st, int B, int H, int d_K, int d_V, int P, float *S, float *Z,
                    void *stream) {
    if (!st) return SATA_EINVAL;
    size_t sb = 0, zb = 0;
    int rc = sata_state_bytes(B, H, d_K, d_V, P, &sb, &zb);
    if (rc) return rc;
    if ((sb && !S) || (zb && !Z)) return SATA_EINVAL;
    if (!aligned16(S) || !aligned16(Z)) return SATA_EALIGN;
    st->B = B;
    st->H = H;
    st->d_K = d_K;
    st->d_V = d_V;
    st->P = P;
    st->F = num_features(d_K, P);
    st->S = S;
    st->Z = Z;
    st->stream = stream;
    st->tokens = 0;
    cudaError_t e = cudaSuccess;
    if (sb) e = cudaMemsetAsync(S, 0, sb, (cudaStream_t)stream);
    if (e == cudaSuccess && zb) e = cudaMemsetAsync(Z, 0, zb, (cudaStream_t)stream);
    return e == cudaSuccess ? SATA_OK : cuda_fail(e);
}

int sata_state_accumulate(sata_state *st, const float *S, const float *Z, int64_t tokens) {
    if (!st || tokens < 0) return SATA_EINVAL;
    size_t sb = 0, zb = 0;
    int rc = sata_state_bytes(st->B, st->H, st->d_K, st->d_V, st->P, &sb, &zb);
    if (rc) return rc;
    if (st->F != num_features(st->d_K, st->P)) return SATA_EINVAL;
    if (sb + zb == 0) {
        st->tokens += tokens;
        return SATA_OK;
    }
    if (!st->S || !st->Z || !S || !Z) return SATA_EINVAL;
    if (!aligned16(st->S) || !aligned16(st->Z) || !aligned16(S) || !aligned16(Z)) return SATA_EALIGN;
    const cudaError_t e = launch_state_add(st->S, st->Z, S, Z, (int64_t)(sb / sizeof(float)),
                                           (int64_t)(zb / sizeof(float)), (cudaStream_t)st->stream);
    if (e != cudaSuccess) return cuda_fail(e);
    st->tokens += tokens;
    return SATA_OK;
}

int sata_workspace_bytes(int B, int H, int64_t N, int d_K, int d_V, int P, size_t *bytes) {
    if (!bytes || N < 0) return SATA_EINVAL;
    int BH = 0;
    int rc = check_heads(B, H, &BH);
    if (rc) return rc;
    rc = check_shape(d_K, d_V, P);
    if (rc) return rc;
    if (g_opt_prefill_path == 2 && !prefill_tc_supported(d_K, d_V, P)) return SATA_EUNSUPPORTED;
    // sized for the larger of the fresh-state and carried-state cases (a fresh state may be
    // carried in the workspace; a carried one may need a copy of its Z)
    const size_t fresh = prefill_ws_bytes(BH, N, d_K, d_V, P, true, nullptr);
    const size_t carried = prefill_ws_bytes(BH, N, d_K, d_V, P, false, nullptr);
    *bytes = fresh > carried ? fresh : carried;
    return SATA_OK;
}

int sata_backward_workspace_bytes(int B, int H, int64_t N, int d_K, int d_V, int P, size_t *bytes) {
    if (!bytes || N < 0) return SATA_EINVAL;
    int BH = 0;
    int rc = check_heads(B, H, &BH);
    if (rc) return rc;
    rc = check_shape(d_K, d_V, P);
    if (rc) return rc;
    bool use_tc = false;
    prefill_ws_bytes(BH, N, d_K, d_V, P, true, &use_tc);
    *bytes = prefill_backward_workspace_bytes(BH, N, num_features(d_K, P), d_K, d_V, P, use_tc);
    return SATA_OK;
}

int sata_prefill_backward(const void *q, const void *k, const void *v, const float *dy, float *dq,
                          float *dk, float *dv, int B, int H, int64_t N, int d_K, int d_V, int P,
                          void *workspace, size_t ws_bytes, void *stream) {
    int BH = 0;
    int rc = check_heads(B, H, &BH);
    if (rc) return rc;
    if (N < 0) return SATA_EINVAL;
    rc = check_shape(d_K, d_V, P);
    if (rc) return rc;
    if (N == 0 || BH == 0) return SATA_OK;
    if (!q || !k || !v || !dy || !dq || !dk || !dv) return SATA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return SATA_EALIGN;
    if (workspace && !aligned16(workspace)) return SATA_EALIGN;
    cudaError_t e = cudaSuccess;
    const DeviceBasis *basis = device_basis(d_K, P, &e);
    if (!basis) return cuda_fail(e);
    int *flags = device_flags(&e);
    if (!flags) return cuda_fail(e);
    bool use_tc = false;   // the forward it recomputes takes the prefill's path
    prefill_ws_bytes(BH, N, d_K, d_V, P, true, &use_tc);
    if (g_opt_prefill_path == 2 && !use_tc) return SATA_EUNSUPPORTED;
    const size_t need = prefill_backward_workspace_bytes(BH, N, basis->F, d_K, d_V, P, use_tc);
    if (workspace) {
        if (ws_bytes < need) return SATA_ENOMEM;
    } else {
        workspace = device_workspace(3, need, &e);
        if (!workspace) {
            g_last_cuda = (int)e;
            return SATA_ENOMEM;
        }
        ws_bytes = need;
    }
    e = launch_prefill_backward(*basis, BH, N, d_V, q, k, v, dy, dq, dk, dv, workspace, ws_bytes, use_tc,
                                flags, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return SATA_OK;
}

int sata_prefill_ex(const void *q, const void *k, const void *v, float *out, int B, int H,
                    int64_t N, int d_K, int d_V, int P, sata_state *st, void *workspace,
                    size_t ws_bytes, void *stream) {
    int BH = 0;
    int rc = check_prefill_args(B, H, N, d_K, d_V, P, st, &BH);
    if (rc) return rc;
    if (N == 0 || BH == 0) return SATA_OK;
    if (!q || !k || !v || !out) return SATA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SATA_EALIGN;
    if (workspace && !aligned16(workspace)) return SATA_EALIGN;

    bool use_tc = false;
    const size_t need = prefill_ws_bytes(BH, N, d_K, d_V, P, st == nullptr, &use_tc);
    cudaError_t e = cudaSuccess;
    const DeviceBasis *basis = device_basis(d_K, P, &e);
    if (!basis) return cuda_fail(e);
    int *flags = device_flags(&e);
    if (!flags) return cuda_fail(e);
    if (workspace) {
        if (ws_bytes < need) return SATA_ENOMEM;
    } else {
        workspace = device_workspace(0, need, &e);
        if (!workspace) {
            g_last_cuda = (int)e;
            return SATA_ENOMEM;
        }
        ws_bytes = need;
    }
    cudaStream_t s = (cudaStream_t)stream;
    float *S = st ? st->S : nullptr;
    float *Z = st ? st->Z : nullptr;
    const bool state_in = st != nullptr;
    e = use_tc ? launch_prefill_tc(*basis, BH, N, d_V, q, k, v, out, S, Z, state_in, workspace,
                                   ws_bytes, flags, s, nullptr)
               : launch_prefill_simt(*basis, BH, N, d_V, q, k, v, out, S, Z, state_in, workspace,
                                     ws_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (st) st->tokens += N;
    return SATA_OK;
}

int sata_prefill_f32(const float *q, const float *k, const float *v, float *out, int B, int H, int64_t N, int d_K,
                     int d_V, int P, sata_state *st, void *stream) {
    int BH = 0;
    int rc = check_prefill_args(B, H, N, d_K, d_V, P, st, &BH);
    if (rc) return rc;
    if (N == 0 || BH == 0) return SATA_OK;
    if (!q || !k || !v || !out) return SATA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SATA_EALIGN;
    const int64_t F = num_features(d_K, P);
    const size_t need = prefill_simt_workspace_bytes(BH, N, F, d_V, st == nullptr);
    cudaError_t e = cudaSuccess;
    const DeviceBasis *basis = device_basis(d_K, P, &e);
    if (!basis) return cuda_fail(e);
    void *workspace = device_workspace(0, need, &e);
    if (!workspace) {
        g_last_cuda = (int)e;
        return SATA_ENOMEM;
    }
    e = launch_prefill_simt(*basis, BH, N, d_V, q, k, v, out, st ? st->S : nullptr, st ? st->Z : nullptr,
                            st != nullptr, workspace, need, (cudaStream_t)stream, nullptr, true);
    if (e != cudaSuccess) return cuda_fail(e);
    if (st) st->tokens += N;
    return SATA_OK;
}

int sata_prefill_host(const void *q, const void *k, const void *v, float *out, int B, int H, int64_t N,
                      int d_K, int d_V, int P, sata_state *st, void *stream) {
    int BH = 0;
    int rc = check_prefill_args(B, H, N, d_K, d_V, P, st, &BH);
    if (rc) return rc;
    if (N == 0 || BH == 0) return SATA_OK;
    if (!q || !k || !v || !out) return SATA_EINVAL;
    bool use_tc = false;
    const size_t need = prefill_ws_bytes(BH, N, d_K, d_V, P, st == nullptr, &use_tc, true);
    cudaError_t e = cudaSuccess;
    const DeviceBasis *basis = device_basis(d_K, P, &e);
    if (!basis) return cuda_fail(e);
    int *flags = device_flags(&e);
    if (!flags) return cuda_fail(e);
    // device copies of the inputs and the output (slot 2), then the prefill workspace (slot 0)
    const size_t nq = (size_t)BH * N * d_K * 2, nv = (size_t)BH * N * d_V * 2, no = (size_t)BH * N * d_V * 4;
    const size_t a16 = 256;
    const size_t oq = 0, ok_ = (oq + nq + a16 - 1) / a16 * a16, ov = (ok_ + nq + a16 - 1) / a16 * a16,
                 oo = (ov + nv + a16 - 1) / a16 * a16, nio = oo + no;
    uint8_t *io_buf = (uint8_t *)device_workspace(2, nio, &e);
    if (!io_buf) {
        g_last_cuda = (int)e;
        return SATA_ENOMEM;
    }
    void *workspace = device_workspace(0, need, &e);
    if (!workspace) {
        g_last_cuda = (int)e;
        return SATA_ENOMEM;
    }
    cudaStream_t s = (cudaStream_t)stream;
    float *S = st ? st->S : nullptr;
    float *Z = st ? st->Z : nullptr;
    const bool state_in = st != nullptr;
    void *dq = io_buf + oq, *dk = io_buf + ok_, *dv = io_buf + ov;
    float *dout = (float *)(io_buf + oo);
    if (use_tc) {
        HostIO io{q, k, v, out, nullptr, nullptr, nullptr};
        if ((e = device_copy_streams(&io.h2d, &io.d2h, &io.aux)) != cudaSuccess) return cuda_fail(e);
        e = launch_prefill_tc(*basis, BH, N, d_V, dq, dk, dv, dout, S, Z, state_in, workspace, need, flags, s, &io);
    } else {   // CUDA-core path: whole copies around the call
        if ((e = cudaMemcpyAsync(dq, q, nq, cudaMemcpyHostToDevice, s)) == cudaSuccess &&
            (e = cudaMemcpyAsync(dk, k, nq, cudaMemcpyHostToDevice, s)) == cudaSuccess &&
            (e = cudaMemcpyAsync(dv, v, nv, cudaMemcpyHostToDevice, s)) == cudaSuccess &&
            (e = launch_prefill_simt(*basis, BH, N, d_V, dq, dk, dv, dout, S, Z, state_in, workspace, need, s)) ==
                cudaSuccess)
            e = cudaMemcpyAsync(out, dout, no, cudaMemcpyDeviceToHost, s);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    if (st) st->tokens += N;
    return SATA_OK;
}

int sata_prefill(const void *q, const void *k, const void *v, float *out, int B, int H, int64_t N,
                 int d_K, int d_V, int P) {
    return sata_prefill_ex(q, k, v, out, B, H, N, d_K, d_V, P, nullptr, nullptr, 0, g_stream);
}

int sata_decode_step(sata_state *st, const void *q, const void *k, const void *v, float *out) {
    if (!st) return SATA_EINVAL;
    int BH = 0;
    int rc = check_heads(st->B, st->H, &BH);
    if (rc) return rc;
    rc = check_shape(st->d_K, st->d_V, st->P);
    if (rc) return rc;
    if (st->F != num_features(st->d_K, st->P)) return SATA_EINVAL;
    if (BH == 0) return SATA_OK;
    if (!q || !k || !v || !out || !st->S || !st->Z) return SATA_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(st->S) ||
        !aligned16(st->Z))
        return SATA_EALIGN;
    cudaError_t e = cudaSuccess;
    const DeviceBasis *basis = device_basis(st->d_K, st->P, &e);
    if (!basis) return cuda_fail(e);
    float *partials =
        (float *)device_workspace(1, decode_workspace_bytes(BH, basis->F, st->d_V), &e);
    if (!partials) {
        g_last_cuda = (int)e;
        return SATA_ENOMEM;
    }
    e = launch_decode(*basis, BH, st->d_V, st->S, st->Z, q, k, v, out, partials,
                      (cudaStream_t)st->stream);
    if (e != cudaSuccess) return cuda_fail(e);
    st->tokens += 1;
    return SATA_OK;
}

int sata_set_option(int key, int64_t value) {
    switch (key) {
        case SATA_OPT_PREFILL_PATH:
            if (value < 0 || value > 2) return SATA_EINVAL;
            g_opt_prefill_path = value;
            return SATA_OK;
        case SATA_OPT_WAIT_LIMIT:
            if (value < 0) return SATA_EINVAL;
            g_opt_wait_limit = value;
            return SATA_OK;
        case SATA_OPT_TEST_STALL:
            g_opt_test_stall = value ? 1 : 0;
            return SATA_OK;
        case SATA_OPT_TIME_KERNELS:
            g_opt_time_kernels = value ? 1 : 0;
            return SATA_OK;
        case SATA_OPT_DETERMINISTIC:
            g_opt_deterministic = value ? 1 : 0;
            return SATA_OK;
        default: return SATA_EINVAL;
    }
}

int sata_get_option(int key, int64_t *value) {
    if (!value) return SATA_EINVAL;
    switch (key) {
        case SATA_OPT_PREFILL_PATH: *value = g_opt_prefill_path; return SATA_OK;
        case SATA_OPT_WAIT_LIMIT: *value = g_opt_wait_limit; return SATA_OK;
        case SATA_OPT_TEST_STALL: *value = g_opt_test_stall; return SATA_OK;
        case SATA_OPT_TIME_KERNELS: *value = g_opt_time_kernels; return SATA_OK;
        case SATA_OPT_DETERMINISTIC: *value = g_opt_deterministic; return SATA_OK;
        default: return SATA_EINVAL;
    }
}

}  // extern "C"
