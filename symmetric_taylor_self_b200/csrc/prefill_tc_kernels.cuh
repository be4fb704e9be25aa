// Tensor-core prefill, host side: the unit plans (which pair tile and slots each CTA
// owns), the workspace plan and the driver that enqueues prep, scan and finish per
// segment (pipelining the copies on the host-buffer path).  The kernels are in
// prefill_tc_prep.cuh, prefill_tc_scan.cuh and prefill_tc_finish.cuh.
#pragma once

#include "prefill_tc_finish.cuh"
#include "prefill_tc_prep.cuh"
#include "prefill_tc_scan.cuh"

namespace sata {
namespace {

// ------------------------------------------------------------------ host ----

// Unit plan: which (pair tile, l values) each CTA owns, and per (unit, slot, row)
// the basis index and C/p! of feature (a, b, l), or -1 / 0 where the row is no
// feature (b > l, degree >= P, or a padding pair).
struct UnitPlan {
    int D = 0, P = 0, NL = 0, NPT = 0, G = 0;
    std::vector<uint16_t> pairs;       // [NPT*128]
    std::vector<int32_t> unit_k, unit_nl, unit_l;   // [G], [G], [G*NL]
    std::vector<float> coef;           // [G*NL*128]
    std::vector<int32_t> fidx;         // [G*NL*128]
    size_t off_k = 0, off_nl = 0, off_l = 0, off_coef = 0, off_fidx = 0, bytes = 0;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// floor(log2 c), c = sqrt(d_K): the largest e with 2^(2e) <= d_K.
int floor_log2_c(int d_K) {
    int e = 0;
    while ((int64_t)1 << (2 * (e + 1)) <= d_K) ++e;
    return e;
}

bool build_unit_plan(int D, int P, int NL, UnitPlan &up) {
    HostBasis hb;
    if (!build_basis_host(D, P, hb)) return false;
    // basis index of each sorted tuple of real indices (indices < D), keyed a | b << 8 | l << 16
    std::map<uint32_t, int32_t> index_of;
    for (size_t f = 0; f < hb.tuples.size(); ++f) {
        uint32_t idx[3] = {(uint32_t)D, (uint32_t)D, (uint32_t)D};
        for (size_t m = 0; m < hb.tuples[f].size(); ++m) idx[m] = hb.tuples[f][m];
        index_of[idx[0] | (idx[1] << 8) | (idx[2] << 16)] = (int32_t)f;
    }
    up.D = D;
    up.P = P;
    up.NL = NL;
    const int npair = (D + 1) * (D + 2) / 2;
    up.NPT = (npair + 127) / 128;
    up.pairs.assign((size_t)up.NPT * 128, (uint16_t)(D | (D << 8)));
    std::vector<int> pa(npair), pb(npair);
    {
        int i = 0;
        for (int b = 0; b <= D; ++b)
            for (int a = 0; a <= b; ++a, ++i) {
                pa[i] = a;
                pb[i] = b;
                up.pairs[i] = (uint16_t)(a | (b << 8));
            }
    }
    struct Unit {
        int k, nl;
        int l[16];
    };
    std::vector<Unit> units;
    int64_t covered = 0;
    for (int k = 0; k < up.NPT; ++k) {
        std::vector<int> ls;
        for (int l = 0; l <= D; ++l) {
            bool any = false;
            for (int r = 0; r < 128 && !any; ++r) {
                const int i = k * 128 + r;
                if (i >= npair || pb[i] > l) continue;
                const int p = (pa[i] < D) + (pb[i] < D) + (l < D);
                any = p < P;
            }
            if (any) ls.push_back(l);
        }
        for (size_t s = 0; s < ls.size(); s += NL) {
            Unit u{k, 0, {}};
            for (size_t j = s; j < ls.size() && j < s + NL; ++j) u.l[u.nl++] = ls[j];
            units.push_back(u);
        }
    }
    std::stable_sort(units.begin(), units.end(), [](const Unit &x, const Unit &y) { return x.nl > y.nl; });
    up.G = (int)units.size();
    up.unit_k.resize(up.G);
    up.unit_nl.resize(up.G);
    up.unit_l.assign((size_t)up.G * NL, D);
    up.coef.assign((size_t)up.G * NL * 128, 0.f);
    up.fidx.assign((size_t)up.G * NL * 128, -1);
    for (int g = 0; g < up.G; ++g) {
        const Unit &u = units[g];
        up.unit_k[g] = u.k;
        up.unit_nl[g] = u.nl;
        for (int j = 0; j < u.nl; ++j) {
            const int l = u.l[j];
            up.unit_l[(size_t)g * NL + j] = l;
            for (int r = 0; r < 128; ++r) {
                const int i = u.k * 128 + r;
                if (i >= npair || pb[i] > l) continue;
                const int p = (pa[i] < D) + (pb[i] < D) + (l < D);
                if (p >= P) continue;
                auto it = index_of.find((uint32_t)pa[i] | ((uint32_t)pb[i] << 8) | ((uint32_t)l << 16));
                if (it == index_of.end()) return false;
                const size_t at = ((size_t)g * NL + j) * 128 + r;
                up.fidx[at] = it->second;
                // C_p / p! = 1 / prod over runs of equal real indices of (run length)!
                up.coef[at] = (float)((double)hb.mult[it->second] / (p == 3 ? 6.0 : (p == 2 ? 2.0 : 1.0)));
                ++covered;
            }
        }
    }
    if (covered != (int64_t)hb.tuples.size()) return false;   // every feature exactly once
    up.off_k = align256((size_t)up.NPT * 128 * sizeof(uint16_t));
    up.off_nl = up.off_k + align256((size_t)up.G * 4);
    up.off_l = up.off_nl + align256((size_t)up.G * 4);
    up.off_coef = up.off_l + align256((size_t)up.G * NL * 4);
    up.off_fidx = up.off_coef + align256(up.coef.size() * 4);
    up.bytes = up.off_fidx + align256(up.fidx.size() * 4);
    return true;
}

std::mutex g_plan_mu;
std::map<std::tuple<int, int, int>, UnitPlan> g_plans;

const UnitPlan *unit_plan(int D, int P, int NL) {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    const auto key = std::make_tuple(D, P, NL);
    auto it = g_plans.find(key);
    if (it != g_plans.end()) return &it->second;
    UnitPlan up;
    if (!build_unit_plan(D, P, NL, up)) return nullptr;
    return &g_plans.emplace(key, std::move(up)).first->second;
}

// Workspace: per-head maxima, the prescaled fp16 rows, the summed readouts of a
// segment (and, in the fixed-order mode only, the per-unit partials), and the
// state between segments when the caller keeps none.  The device-buffer path
// runs as one segment in the default mode; the host-buffer path splits the
// sequence so that copies overlap the kernels; the fixed-order mode splits it
// to bound the partial buffer.
struct Plan {
    const UnitPlan *up = nullptr;
    int G = 1, nchunks = 0, nc_seg = 0, nseg = 0;   // nc_seg: chunks of the longest segment
    // host-buffer path: segment starts (chunks) of a non-uniform split, seg_c0[nseg] = nchunks
    bool profiled = false;
    int seg_c0[kHostSegments + 1] = {};
    // host-buffer path: each segment's prep runs on a side stream ahead of the scans, so
    // the per-head maxima have one buffer per segment
    int nstats = 1;
    size_t stats_bytes = 0;
    size_t off_stats = 0, off_q16 = 0, off_k16 = 0, off_v16 = 0, off_red = 0, off_part = 0, off_state = 0,
           total = 0;
};

template <int DK, int DV>
bool make_plan(int BH, int64_t N, int64_t F, int P, bool need_state, int min_segments, bool deterministic,
               Plan &pl) {
    using C = Cfg<DK, DV>;
    const UnitPlan *up = unit_plan(DK, P, C::NL);
    if (!up) return false;
    pl.up = up;
    pl.G = up->G;
    pl.nchunks = (int)((N + kL - 1) / kL);
    int64_t nseg = min_segments;
    if (deterministic) {
        const size_t per_chunk = (size_t)BH * pl.G * sum_quads(DV) * kL * 16;
        int64_t seg = (int64_t)(kPartialBudget / per_chunk);
        if (seg < 1) seg = 1;
        const int64_t need = (pl.nchunks + seg - 1) / seg;
        if (need > nseg) nseg = need;
    }
    if (nseg > pl.nchunks) nseg = pl.nchunks;
    if (nseg < 1) nseg = 1;
    pl.nc_seg = (int)((pl.nchunks + nseg - 1) / nseg);
    pl.nseg = (pl.nchunks + pl.nc_seg - 1) / pl.nc_seg;
    if (!deterministic && min_segments == kHostSegments && pl.nchunks >= 16 * kHostSegments) {
        // Copies pipelined with the kernels: the first segment's inputs and the last one's
        // output are exposed, so those segments are short.  A segment's inputs copy in about
        // a third of its compute time and its output in about a quarter, so each segment can
        // be a few times its predecessor while its inputs still land in time, and the last a
        // fraction of the one before it.  8 %, 18 %, 62 %, 12 % of the chunks measured best of
        // the splits tried once the segments' own costs had come down (2.6 % faster end to end
        // at 65536 tokens than 10/20/55/15, which had been best before; uniform quarters were
        // 4 % slower than that).
        static_assert(kHostSegments == 4, "split profile");
        const int cum[kHostSegments] = {0, 8, 26, 88};
        for (int i = 0; i < kHostSegments; ++i) pl.seg_c0[i] = (int)((int64_t)pl.nchunks * cum[i] / 100);
        pl.seg_c0[kHostSegments] = pl.nchunks;
        pl.profiled = true;
        pl.nseg = kHostSegments;
        pl.nc_seg = 0;
        for (int i = 0; i < kHostSegments; ++i)
            if (pl.seg_c0[i + 1] - pl.seg_c0[i] > pl.nc_seg) pl.nc_seg = pl.seg_c0[i + 1] - pl.seg_c0[i];
    }
    const bool piped = !deterministic && min_segments == kHostSegments;
    pl.nstats = piped ? pl.nseg : 1;
    pl.stats_bytes = align256((size_t)BH * 4 * sizeof(float));
    pl.off_stats = 0;
    pl.off_q16 = pl.nstats * pl.stats_bytes;
    const size_t rows = (size_t)BH * pl.nchunks * kL;   // whole chunks, chunk-interleaved
    pl.off_k16 = pl.off_q16 + align256(rows * DK * 2);
    pl.off_v16 = pl.off_k16 + align256(rows * DK * 2);
    pl.off_red = pl.off_v16 + align256(rows * DV * 2);
    pl.off_part = pl.off_red + align256((size_t)BH * sum_quads(DV) * kL * 16 * pl.nc_seg);
    pl.off_state = pl.off_part +
                   (deterministic ? align256((size_t)BH * pl.G * sum_quads(DV) * kL * 16 * pl.nc_seg) : 0);
    pl.total = pl.off_state + (need_state && pl.nseg > 1 ? align256((size_t)BH * F * (DV + 1) * sizeof(float)) : 0);
    return true;
}

// Enqueue the copy of token rows [t0, t1) of a [BH][N][width] tensor (elem bytes each).
cudaError_t copy_rows(void *dst, const void *src, int BH, int64_t N, int64_t t0, int64_t t1, int width, int elem,
                      cudaMemcpyKind kind, cudaStream_t s) {
    const size_t pitch = (size_t)N * width * elem, off = (size_t)t0 * width * elem;
    return cudaMemcpy2DAsync((uint8_t *)dst + off, pitch, (const uint8_t *)src + off, pitch,
                             (size_t)(t1 - t0) * width * elem, BH, kind, s);
}

// dvs, voff: v, out and a caller's S have rows of dvs values, of which this call covers
// the DV columns from voff on (dvs = DV, voff = 0: whole rows).  The caller's Z is
// written whole by every such call.  Not with host buffers.
template <int DK, int DV>
cudaError_t run(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k, const void *v,
                float *out, float *S, float *Z, bool state_in, void *ws, size_t ws_bytes, int *flags,
                cudaStream_t stream, const HostIO *io, float *den_out, int dvs = DV, int voff = 0) {
    using C = Cfg<DK, DV>;
    const int64_t F = basis.F;
    const bool own_state = (S == nullptr);
    if (dvs < DV || voff < 0 || voff + DV > dvs || dvs % 8 != 0 || voff % 8 != 0 || (io && dvs != DV))
        return cudaErrorInvalidValue;
    const int s_ld = own_state ? DV : dvs, s_off = own_state ? 0 : voff;   // the state's rows
    const int min_seg = io ? kHostSegments : 1;
    const bool det = g_opt_deterministic != 0;
    Plan pl;
    if (!make_plan<DK, DV>(BH, N, F, basis.P, own_state, min_seg, det, pl)) return cudaErrorInvalidValue;
    if (ws_bytes < pl.total) return cudaErrorInvalidValue;
    const UnitPlan &up = *pl.up;
    cudaError_t e = cudaSuccess;
    const uint8_t *tab = (const uint8_t *)device_table(
        ((uint64_t)DK << 32) | ((uint64_t)basis.P << 16) | (uint64_t)up.NL | (uint64_t(1) << 60), up.bytes,
        [&up](uint8_t *h) {
            std::memcpy(h, up.pairs.data(), up.pairs.size() * sizeof(uint16_t));
            std::memcpy(h + up.off_k, up.unit_k.data(), up.unit_k.size() * 4);
            std::memcpy(h + up.off_nl, up.unit_nl.data(), up.unit_nl.size() * 4);
            std::memcpy(h + up.off_l, up.unit_l.data(), up.unit_l.size() * 4);
            std::memcpy(h + up.off_coef, up.coef.data(), up.coef.size() * 4);
            std::memcpy(h + up.off_fidx, up.fidx.data(), up.fidx.size() * 4);
        },
        &e);
    if (!tab) return e != cudaSuccess ? e : cudaErrorMemoryAllocation;
    uint8_t *w = (uint8_t *)ws;
    __half *q16 = (__half *)(w + pl.off_q16), *k16 = (__half *)(w + pl.off_k16), *v16 = (__half *)(w + pl.off_v16);
    float *part = (float *)(w + pl.off_part);
    const int nseg = pl.nseg;
    if (own_state && nseg > 1) {
        S = (float *)(w + pl.off_state);
        Z = S + (size_t)BH * F * DV;
    }
    const float inv_c = 1.0f / sqrtf((float)DK);
    const auto *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k, *vb = (const __nv_bfloat16 *)v;

    e = cudaFuncSetAttribute(tc_scan_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_finish_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             FinCfg<DK, DV>::SMEM);
    if (e != cudaSuccess) return e;
    int stall = -1;
    if (g_opt_test_stall) {
        stall = pl.nchunks > 1 ? 1 : 0;
        g_opt_test_stall = 0;
    }
    const int64_t wait_ns = g_opt_wait_limit > 0 ? g_opt_wait_limit : kDefaultWaitNs;
    // events of the host-buffer pipeline; released once enqueued (they live until they complete)
    std::vector<cudaEvent_t> events;
    auto new_event = [&events](cudaEvent_t *ev) {
        cudaError_t r = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (r == cudaSuccess) events.push_back(*ev);
        return r;
    };
    struct Release {
        std::vector<cudaEvent_t> &ev;
        ~Release() { for (cudaEvent_t x : ev) cudaEventDestroy(x); }
    } release{events};
    // Host buffers (not in the fixed-order mode): each segment's maxima and prescaled rows are
    // built on the side stream `ps` as soon as its rows have landed, so they run beside the
    // previous segment's scan (in its last wave, where SMs fall idle) instead of between
    // the scans; a segment's maxima have their own buffer.  The incoming-state bound, the
    // scans and the finishes stay on `stream`, in order.  (A finish on the side stream
    // competed with the next scan's first wave for SMs and gained little.)
    const bool piped = io && !det;
    cudaStream_t ps = piped ? io->aux : stream;
    if (io) {   // the copies follow the work already on `stream` (an earlier call may still read these buffers)
        cudaEvent_t ev;
        if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, stream)) || (e = cudaStreamWaitEvent(io->h2d, ev, 0)) ||
            (e = cudaStreamWaitEvent(io->d2h, ev, 0)) || (piped && (e = cudaStreamWaitEvent(ps, ev, 0))))
            return e;
    }
    float *red = (float *)(w + pl.off_red);
    for (int s = 0; s < nseg; ++s) {
        const int c0s = pl.profiled ? pl.seg_c0[s] : s * pl.nc_seg;
        const int ncs = pl.profiled ? pl.seg_c0[s + 1] - c0s
                                    : ((pl.nchunks - c0s < pl.nc_seg) ? pl.nchunks - c0s : pl.nc_seg);
        const int64_t tok0 = (int64_t)c0s * kL, tok1 = (int64_t)(c0s + ncs) * kL < N ? (int64_t)(c0s + ncs) * kL : N;
        float *stats = (float *)(w + pl.off_stats + (size_t)(piped ? s : 0) * pl.stats_bytes);
        if (io) {   // this segment's inputs: host -> device on the copy stream; its prep waits for them
            cudaEvent_t ev;
            if ((e = copy_rows((void *)q, io->q, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)k, io->k, BH, N, tok0, tok1, DK, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = copy_rows((void *)v, io->v, BH, N, tok0, tok1, DV, 2, cudaMemcpyHostToDevice, io->h2d)) ||
                (e = new_event(&ev)) || (e = cudaEventRecord(ev, io->h2d)) || (e = cudaStreamWaitEvent(ps, ev, 0)))
                return e;
        }
        const bool load_state = (s > 0 || state_in);
        {   // this segment's maxima and prescaled rows (on ps), then the incoming-state bound
            if ((e = cudaMemsetAsync(stats, 0, (size_t)BH * 4 * sizeof(float), ps)) != cudaSuccess) return e;
            const int64_t ntok = tok1 - tok0;
            int bx = (int)((ntok * (DK / 8) + 255) / 256);
            const int bmax = (148 * 8 + BH - 1) / BH;
            if (bx > bmax) bx = bmax;
            if (bx < 1) bx = 1;
            launch_begin(kTcStats, ps);
            tc_stats_kernel<DK, DV><<<(unsigned)((int64_t)bx * BH), 256, 0, ps>>>(qb, kb, vb, stats, N, tok0, tok1, bx,
                                                                                dvs);
            launch_end(kTcStats, ps);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            {
                const int64_t nwork = (int64_t)BH * ntok;   // one thread per token row
                const int pgrid = (int)((nwork + 255) / 256 < 148 * 16 ? (nwork + 255) / 256 : 148 * 16);
                launch_begin(kTcPrep, ps);
                tc_prep_kernel<DK, DV><<<pgrid, 256, 0, ps>>>(qb, kb, vb, stats, q16, k16, v16, BH, N, tok0, tok1,
                                                               pl.nchunks, flags, dvs, voff);
                launch_end(kTcPrep, ps);
            }
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            if (piped) {
                cudaEvent_t ev;
                if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, ps)) || (e = cudaStreamWaitEvent(stream, ev, 0)))
                    return e;
            }
            if (load_state) {
                int ny = (148 * 8 + BH - 1) / BH;   // about eight blocks per SM over all heads
                ny = ny < 8 ? 8 : (ny > 1024 ? 1024 : ny);
                launch_begin(kTcStateStats, stream);
                tc_state_stats_kernel<<<dim3(BH, ny), 256, 0, stream>>>(S, Z, stats, F, s_ld);
                launch_end(kTcStateStats, stream);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
        }
        ScanParams sp;
        sp.q16 = q16;
        sp.k16 = k16;
        sp.v16 = v16;
        sp.stats = stats;
        sp.pairs = (const uint16_t *)tab;
        sp.unit_k = (const int32_t *)(tab + up.off_k);
        sp.unit_nl = (const int32_t *)(tab + up.off_nl);
        sp.unit_l = (const int32_t *)(tab + up.off_l);
        sp.unit_coef = (const float *)(tab + up.off_coef);
        sp.unit_fidx = (const int32_t *)(tab + up.off_fidx);
        sp.S = S;
        sp.Z = Z;
        sp.s_ld = s_ld;
        sp.s_off = s_off;
        if (!det && (e = cudaMemsetAsync(red, 0, (size_t)BH * ncs * sum_quads(DV) * kL * 16, stream)) !=
                        cudaSuccess)
            return e;
        sp.part = det ? part : red;
        sp.red_atomic = det ? 0 : 1;
        sp.flags = flags;
        sp.F = F;
        sp.N = N;
        sp.BH = BH;
        sp.G = pl.G;
        sp.c0 = c0s;
        sp.nc = ncs;
        sp.nch = pl.nchunks;
        sp.P = basis.P;
        sp.load_state = load_state ? 1 : 0;
        sp.store_state = (s + 1 < nseg || !own_state) ? 1 : 0;
        sp.stall_chunk = stall;
        sp.inv_c = inv_c;
        sp.lc = floor_log2_c(DK);
        sp.wait_ns = wait_ns;
        launch_begin(kTcScan, stream);
        tc_scan_kernel<DK, DV><<<BH * pl.G, kScanThreads, C::SMEM, stream>>>(sp);
        launch_end(kTcScan, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (det) {   // the units' partials summed in a fixed order
            const int64_t rwork = (int64_t)BH * ncs * sum_quads(DV) * kL;
            launch_begin(kTcReduce, stream);
            tc_reduce_kernel<DV><<<(int)((rwork + 255) / 256 < 148 * 32 ? (rwork + 255) / 256 : 148 * 32), 256, 0,
                                   stream>>>((const float4 *)part, (float4 *)red, BH, pl.G, ncs);
            launch_end(kTcReduce, stream);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        launch_begin(kTcFinish, stream);
        tc_finish_kernel<DK, DV><<<(int)((int64_t)BH * ncs), 256, FinCfg<DK, DV>::SMEM, stream>>>(
            q16, k16, v16, stats, red, out, den_out, c0s, ncs, pl.nchunks, N, basis.P, inv_c, flags, wait_ns, dvs,
            voff);
        launch_end(kTcFinish, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (io) {   // this segment's output: device -> host on the second copy stream
            cudaEvent_t ev;
            if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, stream)) || (e = cudaStreamWaitEvent(io->d2h, ev, 0)) ||
                (e = copy_rows(io->out, out, BH, N, tok0, tok1, DV, 4, cudaMemcpyDeviceToHost, io->d2h)))
                return e;
        }
    }
    if (io) {   // the caller's stream completes after the last copy back
        cudaEvent_t ev;
        if ((e = new_event(&ev)) || (e = cudaEventRecord(ev, io->d2h)) || (e = cudaStreamWaitEvent(stream, ev, 0)))
            return e;
    }
    return cudaSuccess;
}

}  // namespace

// Non-template entry points of one (d_K, d_V) instance (declared in prefill_tc_shapes.h).
#define SATA_TC_DEFINE(a, b)                                                                                  \
    size_t tc_workspace_##a##_##b(int BH, int64_t N, int64_t F, int P, bool need_state, int min_seg, bool det) { \
        Plan pl;                                                                                              \
        return make_plan<a, b>(BH, N, F, P, need_state, min_seg, det, pl) ? pl.total : 0;                     \
    }                                                                                                         \
    cudaError_t tc_run_##a##_##b(const DeviceBasis &basis, int BH, int64_t N, const void *q, const void *k,   \
                                 const void *v, float *out, float *S, float *Z, bool state_in, void *ws,       \
                                 size_t ws_bytes, int *flags, cudaStream_t stream, const HostIO *io,          \
                                 float *den_out, int dvs, int voff) {                                         \
        return run<a, b>(basis, BH, N, q, k, v, out, S, Z, state_in, ws, ws_bytes, flags, stream, io, den_out,   \
                         dvs, voff);                                                                          \
    }

}  // namespace sata
