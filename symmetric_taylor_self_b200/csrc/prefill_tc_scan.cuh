// Tensor-core prefill, the scan: the warp-specialised kernel that updates the TMEM state
// and reads it out per chunk (prefill and gradient scans), with its drains and conversion.
#pragma once

#include "prefill_tc_common.cuh"

namespace sata {
namespace {

// ----------------------------------------------------------------- scan ----

// Token row t of chunk cl into registers, with x~_l of each slot (half2 broadcasts).
template <int DK, int NX, int NL>
__device__ __forceinline__ void fetch_row(const __half *x16, const ScanParams &p, int64_t bh, const int *sl, int cl,
                                          int t, uint32_t (&x)[NX], uint32_t (&xl)[NL]) {
    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
    const uint4 *cr = chunk_rows<DK>(x16, bh, p.nch, p.c0 + cl);
    load_row<DK>(cr, t, valid, x);
#pragma unroll
    for (int s = 0; s < NL; ++s) xl[s] = row_half2(cr, t, sl[s], DK, valid);
}

// q side: readout R of chunk cl (TMEM, this warp's lanes), combined over the slots with
// q~_l, scaled to the true frame and added into the head's sums (or written as this
// unit's partial).  Arrives on rf_bar once every column is read.
template <int DK, int DV>
__device__ __forceinline__ void q_drain(const ScanParams &p, int64_t bh, int64_t part_base, int nl, int e_ms, int E,
                                        int ev, int cl, int e_tok, int t, int lane, uint32_t tm, uint32_t rf_bar,
                                        const float (&qv)[Cfg<DK, DV>::NL]) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    tc_after();
    const int sg = state_sigma(e_tok, e_ms, E, p.P, p.lc);
    const float upv = pow2f_sat(sg + ev), upz = pow2f_sat(sg);
    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
    constexpr int DQ = sum_quads(DV);
    float4 *dst = reinterpret_cast<float4 *>(p.part) + (part_base + cl) * DQ * kL + t;
    float den = 0.f;
    {
        uint32_t rz[16];
        tc_ld16(tm + C::COL_R + nl * DV, rz);
        tc_wait_ld();
#pragma unroll
        for (int s = 0; s < NL; ++s)
            if (s < nl) den = fmaf(qv[s], __uint_as_float(rz[s]), den);
    }
    // 32 columns at a time (16 when d_V = 16): one load per slot, combined, then the columns'
    // quads added (or stored)
    constexpr int GW = DV >= 32 ? 32 : 16;
#pragma unroll 1
    for (int g = 0; g < DV / GW; ++g) {
        float acc[GW];
#pragma unroll
        for (int i = 0; i < GW; ++i) acc[i] = 0.f;
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            if (s < nl) {
                uint32_t ra[GW];
                if constexpr (GW == 32) tc_ld32(tm + C::COL_R + s * DV + GW * g, ra);
                else tc_ld16(tm + C::COL_R + s * DV + GW * g, ra);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < GW; ++i) acc[i] = fmaf(qv[s], __uint_as_float(ra[i]), acc[i]);
            }
        }
        if (g == DV / GW - 1) {   // every column read: the next readout may overwrite R
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(rf_bar);
        }
        if (valid) {
#pragma unroll
            for (int i4 = 0; i4 < GW / 4; ++i4) {
                const float4 val = make_float4(acc[4 * i4] * upv, acc[4 * i4 + 1] * upv, acc[4 * i4 + 2] * upv,
                                               acc[4 * i4 + 3] * upv);
                if (p.red_atomic) atomicAdd(dst + (GW / 4 * g + i4) * kL, val);
                else dst[(GW / 4 * g + i4) * kL] = val;
            }
        }
    }
    if (valid) {   // the Z column opens the last quad (its other columns are padding)
        const float4 val = make_float4(den * upz, 0.f, 0.f, 0.f);
        if (p.red_atomic) atomicAdd(dst + (DV / 4) * kL, val);
        else dst[(DV / 4) * kL] = val;
    }
}

// Gradient scan (JAC) drain: R of chunk cl holds, per slot s (index i_s) and column j,
// sum_pairs P2(a_t) B[pair, (s, j)]; the token's output for slot s is its contraction with
// the token's multipliers m_t (fp32, true frame): sum_{j < d_V} m_t[j] R[t, (s, j)] +
// m_t[d_V] R[t, Z_s], added into sums[bh][i_s][token].  Arrives on rf_bar once every column
// is read.
template <int DK, int DV>
__device__ __forceinline__ void q_drain_jac(const ScanParams &p, int64_t bh, int nl, int E, int ek, int ev, int cl,
                                            int e_tok, int t, int lane, uint32_t tm, uint32_t rf_bar, const int *sl) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    tc_after();
    const int sg = jac_sigma(e_tok, E, ek, p.P, p.lc);
    const float upv = pow2f_sat(sg + ev), upz = pow2f_sat(sg + (p.zscaled ? ev : 0));
    const int64_t tok = (int64_t)(p.c0 + cl) * kL + t;
    const bool valid = tok < p.N;
    // 32 consecutive tokens read 512 contiguous bytes per quad
    const float4 *m4 = reinterpret_cast<const float4 *>(p.mult) + ((int64_t)bh * p.nch + p.c0 + cl) * p.mult_quads * kL + t;
    float acc[NL], accz[NL];
    {
        uint32_t rz[16];
        tc_ld16(tm + C::COL_R + nl * DV, rz);
        tc_wait_ld();
        const float mz = valid ? __ldg(m4 + (DV / 4) * kL).x : 0.f;
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            acc[s] = 0.f;
            accz[s] = mz * __uint_as_float(rz[s]);
        }
    }
    constexpr int GW = DV >= 32 ? 32 : 16;
#pragma unroll 1
    for (int g = 0; g < DV / GW; ++g) {
        float mv[GW];
#pragma unroll
        for (int i4 = 0; i4 < GW / 4; ++i4) {
            const float4 x = valid ? __ldg(m4 + (GW / 4 * g + i4) * kL) : make_float4(0.f, 0.f, 0.f, 0.f);
            mv[4 * i4] = x.x;
            mv[4 * i4 + 1] = x.y;
            mv[4 * i4 + 2] = x.z;
            mv[4 * i4 + 3] = x.w;
        }
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            if (s < nl) {
                uint32_t ra[GW];
                if constexpr (GW == 32) tc_ld32(tm + C::COL_R + s * DV + GW * g, ra);
                else tc_ld16(tm + C::COL_R + s * DV + GW * g, ra);
                tc_wait_ld();
                float a = acc[s];
#pragma unroll
                for (int i = 0; i < GW; ++i) a = fmaf(mv[i], __uint_as_float(ra[i]), a);
                acc[s] = a;
            }
        }
        if (g == DV / GW - 1) {   // every column read: the next readout may overwrite R
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(rf_bar);
        }
    }
    if (valid) {
#pragma unroll
        for (int s = 0; s < NL; ++s)
            if (s < nl) atomicAdd(p.sums_jac + (bh * DK + sl[s]) * p.N + tok, fmaf(acc[s], upv, accz[s] * upz));
    }
}

// conversion: 16 fp32 state columns of one slot's V part -> 8 packed fp16 words, scaled by f.
__device__ __forceinline__ void conv_v(const uint32_t (&rr)[16], float f, uint32_t (&hp)[8]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const __half2 h = __floats2half2_rn(__uint_as_float(rr[2 * w]) * f, __uint_as_float(rr[2 * w + 1]) * f);
        hp[w] = *reinterpret_cast<const uint32_t *>(&h);
    }
}
// conversion: the Z group (column s = Z of slot s, s < nl; padding after) -> 8 packed words.
template <int NL>
__device__ __forceinline__ void conv_z(const uint32_t (&rr)[16], int nl, const float (&sc)[NL], uint32_t (&hp)[8]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int s0 = 2 * w, s1 = 2 * w + 1;
        const float f0 = s0 < nl ? sel(sc, s0) : 0.f;
        const float f1 = s1 < nl ? sel(sc, s1) : 0.f;
        const __half2 h = __floats2half2_rn(__uint_as_float(rr[2 * w]) * f0, __uint_as_float(rr[2 * w + 1]) * f1);
        hp[w] = *reinterpret_cast<const uint32_t *>(&h);
    }
}

// JAC = false: the prefill scan (features of degree < P, den from the Z columns).
// JAC = true: a gradient scan of the backward pass: pair rows of degree <= P - 2 (the
// derivative T_{P-1} of the Taylor weight), slots index the key-side vector as a value
// dimension, the Z columns take zval16 (or 1), and the drain contracts each slot's
// columns with the token's multipliers (q_drain_jac).  Fresh state only.
template <int DK, int DV, bool JAC = false>
__global__ void __launch_bounds__(kScanThreads, 1) tc_scan_kernel(const ScanParams p) {
    using C = Cfg<DK, DV>;
    constexpr int NL = C::NL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto BAR = [bar0](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *sl = reinterpret_cast<int *>(smem + C::OFF_L);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // head-major order (a head's units, largest first, then the next head's): the CTAs
    // resident at a time share one or two heads' token rows and sums in L2
    const int64_t bh = blockIdx.x / p.G;
    const int u = blockIdx.x % p.G;
    const int ktile = p.unit_k[u];
    const int nl = p.unit_nl[u];
    const int NU = (nl * (DV + 1) + 15) / 16 * 16;   // MMA N of this unit
    const HeadExp he = head_exps(p.stats + bh * 4);
    const int E = he.eq + he.ek;
    const float ms = p.stats[bh * 4 + 3];
    const int e_ms = (p.load_state && ms > 0.f)
                         ? scale_exp(ms) + ((p.P - 1) * -he.ek > 0 ? (p.P - 1) * -he.ek : 0) + (he.ev < 0 ? -he.ev : 0)
                         : -1000;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::N_BAR; ++i) {
            uint32_t cnt = 1;
            if (i == C::B_AKF || i == C::B_SR || i == C::B_BSF || i == C::B_BSF + 1 || i == C::B_AQF ||
                i == C::B_RF)
                cnt = 4;

            mbar_init(BAR(i), cnt);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x < NL) sl[threadIdx.x] = p.unit_l[u * NL + threadIdx.x];
    if (warp == kWarpI) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32((const void *)tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_before();
    }
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const Waiter W{abort_flag, p.flags + kFlagTimeout, p.wait_ns};

    if (warp == kWarpI) {
        // ------------------------------------------------ MMA issue (one thread, two chains)
        // The update of chunk cu and the readout of chunk cr (cr < cu: a readout follows its
        // chunk's update) are issued as soon as their operands are ready, whichever is ready
        // first, so the update of chunk c + 1 need not wait behind the readout of chunk c (the
        // drain of chunk c - 1 gates that readout).  No tested barrier can be a phase ahead of
        // its test: each one's next phase needs an MMA this thread has not issued yet.  With
        // nothing ready the thread sleeps briefly; no progress for the wait limit aborts as a
        // blocking wait would.  (1.7 % faster than issuing both chains in chunk order for the
        // prefill; the gradient scans, whose drain contracts every slot separately, ran 2.5 %
        // slower with it and issue in chunk order.)
        if (lane == 0 && JAC) {
            const uint32_t id_u = idesc_f16(128, NU, 1, 1);   // A, B MN-major in shared memory
            const uint32_t id_r = idesc_f16(128, NU, 0, 1);   // A in TMEM, B MN-major
            const uint32_t wb = sb + C::OFF_W;
            bool ok = true;
            for (int cl = 0; cl < p.nc && ok; ++cl) {
                const int b = cl & 1;
                ok = W.wait(BAR(C::B_AKF), cl & 1) && W.wait(BAR(C::B_SR), cl & 1);
                if (!ok) break;
                tc_after();
                const uint32_t ak = sb + C::OFF_AK + b * C::AK_BYTES;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(tmem + C::COL_S, sdesc(ak + ks * 2048, 16384, 1024, 2),
                           sdesc(wb + ks * 2 * C::LBO, C::LBO, 128, 0), id_u,
                           (p.load_state || cl > 0 || ks > 0) ? 1u : 0u);
                tc_commit(BAR(C::B_AKE + b));
                tc_commit(BAR(C::B_UD));
                ok = W.wait(BAR(C::B_AQF), cl & 1) && W.wait(BAR(C::B_BSF + b), (cl >> 1) & 1) &&
                     (cl == 0 || W.wait(BAR(C::B_RF), (cl - 1) & 1));
                if (!ok) break;
                tc_after();
                const uint32_t bs = sb + C::OFF_BS + b * C::W_BYTES;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma_ta(tmem + C::COL_R, tmem + C::COL_AQ + ks * 8,
                              sdesc(bs + ks * 2 * C::LBO, C::LBO, 128, 0), id_r, ks > 0 ? 1u : 0u);
                tc_commit(BAR(C::B_BSE + b));
                tc_commit(BAR(C::B_RD));
            }
            // every issued MMA completes before TMEM is released
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        } else if (lane == 0) {
            const uint32_t id_u = idesc_f16(128, NU, 1, 1);   // A, B MN-major in shared memory
            const uint32_t id_r = idesc_f16(128, NU, 0, 1);   // A in TMEM, B MN-major
            const uint32_t wb = sb + C::OFF_W;
            int cu = 0, cr = 0;
            int64_t t_last = gtimer();
            while (cr < p.nc) {
                bool prog = false;
                if (cu < p.nc && mbar_test(BAR(C::B_AKF), cu & 1) && mbar_test(BAR(C::B_SR), cu & 1)) {
                    const int cl = cu++, b = cl & 1;
                    tc_after();
                    // update: [S|Z] (+)= P2(K)^T [128 pairs x 128 t] . W [128 t x NU]
                    const uint32_t ak = sb + C::OFF_AK + b * C::AK_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma(tmem + C::COL_S, sdesc(ak + ks * 2048, 16384, 1024, 2),
                               sdesc(wb + ks * 2 * C::LBO, C::LBO, 128, 0), id_u,
                               (p.load_state || cl > 0 || ks > 0) ? 1u : 0u);
                    tc_commit(BAR(C::B_AKE + b));
                    tc_commit(BAR(C::B_UD));
                    prog = true;
                }
                if (cr < cu && mbar_test(BAR(C::B_AQF), cr & 1) && mbar_test(BAR(C::B_BSF + (cr & 1)), (cr >> 1) & 1) &&
                    (cr == 0 || mbar_test(BAR(C::B_RF), (cr - 1) & 1))) {
                    const int cl = cr++, b = cl & 1;
                    tc_after();
                    // readout: R = P2(Q) [128 t x 128 pairs] . B [128 pairs x NU]
                    const uint32_t bs = sb + C::OFF_BS + b * C::W_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma_ta(tmem + C::COL_R, tmem + C::COL_AQ + ks * 8,
                                  sdesc(bs + ks * 2 * C::LBO, C::LBO, 128, 0), id_r, ks > 0 ? 1u : 0u);
                    tc_commit(BAR(C::B_BSE + b));
                    tc_commit(BAR(C::B_RD));
                    prog = true;
                }
                if (prog) {
                    t_last = gtimer();
                } else {
                    if (*abort_flag) break;
                    if (gtimer() - t_last > W.limit) {
                        *abort_flag = 1;
                        atomicExch(W.gflag, 1);
                        break;
                    }
                    __nanosleep(40);
                }
            }
            // every issued MMA completes before TMEM is released
            tc_commit(BAR(C::B_FIN));
            W.drain(BAR(C::B_FIN), 0);
        }
    } else if (warp < kWarpQ0) {
        // ------------------------------------------------ k side: P2(k) and W per chunk
        const int t = (warp - kWarpK0) * 32 + lane;
        // Per chunk: P2(k) from the prefetched k row once its buffer is free, then the v row is
        // requested and lands while the update of the previous chunk completes, then W, then
        // the next chunk's k row is requested.
        uint32_t x[C::XW], kl[NL];   // this chunk's k row and k~_l (half2 broadcasts), prefetched
        if (p.nc > 0) fetch_row<DK>(p.k16, p, bh, sl, 0, t, x, kl);
        bool ok = true;
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int b = cl & 1;
            // P2(k) into its double buffer once the update of chunk cl-2 has read it
            if (cl >= 2 && !(ok = W.wait(BAR(C::B_AKE + b), ((cl >> 1) - 1) & 1))) break;
            p2k_dispatch<DK>(ktile, x, smem + C::OFF_AK + b * C::AK_BYTES, t,
                             std::make_integer_sequence<int, C::NPT>{});
            uint4 vr[DV / 8];
            {
                const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
                const uint4 *vcr = chunk_rows<DV>(p.v16, bh, p.nch, p.c0 + cl);
#pragma unroll
                for (int i = 0; i < DV / 8; ++i) vr[i] = valid ? __ldg(vcr + i * 128 + t) : make_uint4(0, 0, 0, 0);
            }
            // W (single buffer) once the update of chunk cl-1 has completed
            if (cl >= 1 && !(ok = W.wait(BAR(C::B_UD), (cl - 1) & 1))) break;
            // W row t: [k~_l0 v | k~_l1 v | ... | k~_l0 k~_l1 ... 0 ...] as 16-byte chunks of 8 columns
            uint8_t *wrow = smem + C::OFF_W + (t >> 3) * C::LBO + (t & 7) * 16;
#pragma unroll
            for (int s = 0; s < NL; ++s) {
                if (s < nl) {
#pragma unroll
                    for (int i = 0; i < DV / 8; ++i)
                        *reinterpret_cast<uint4 *>(wrow + (s * (DV / 8) + i) * 128) = hmul2x4(vr[i], kl[s]);
                }
            }
            uint32_t zv = 0x3C003C00u;   // the Z columns' factor: 1, or the token's value (JAC)
            if constexpr (JAC) {
                if (p.zval16) {
                    const bool valid = (int64_t)(p.c0 + cl) * kL + t < p.N;
                    const uint32_t h =
                        valid ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.zval16) +
                                                ((int64_t)bh * p.nch + p.c0 + cl) * kL + t)
                              : 0u;
                    zv = h | (h << 16);
                }
            }
            for (int z8 = nl * (DV / 8); z8 < NU / 8; ++z8) {
                uint32_t w4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int s0 = z8 * 8 - nl * DV + 2 * j, s1 = s0 + 1;
                    uint32_t lo = 0, hi = 0;
#pragma unroll
                    for (int s = 0; s < NL; ++s) {
                        const uint32_t kz = JAC ? hmul2u(kl[s], zv) : kl[s];
                        lo = (s == s0 && s < nl) ? (kz & 0xFFFFu) : lo;
                        hi = (s == s1 && s < nl) ? (kz & 0xFFFFu) : hi;
                    }
                    w4[j] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4 *>(wrow + z8 * 128) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async();
            __syncwarp();
            // test hook: one producer signal withheld, so the issuer's wait expires
            if (lane == 0 && !(warp == kWarpK0 && p.c0 + cl == p.stall_chunk)) mbar_arrive(BAR(C::B_AKF));
            // the next chunk's k row, requested after the signal: its slot values are used as
            // soon as they land, so the load latency would otherwise sit before the update
            if (cl + 1 < p.nc) fetch_row<DK>(p.k16, p, bh, sl, cl + 1, t, x, kl);
        }
    } else if (warp < kWarpC0) {
        // ------------------------------------------------ q side: P2(q) operand, readout drain
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;               // token row of the chunk = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int64_t part_base = p.red_atomic ? (int64_t)bh * p.nc : ((int64_t)bh * p.G + u) * p.nc;
        uint32_t pq[64], xl[NL];
        float qlp[NL];
        float cum = 0.f;   // column maxima of the chunks before the one drained next
        bool ok = true;
        if (p.nc > 0) {
            uint32_t x[C::XW];
            fetch_row<DK>(p.q16, p, bh, sl, 0, t, x, xl);
            p2q_dispatch<DK, 0, C::NPT>(ktile, x, pq);
        }
        for (int cl = 0; cl < p.nc; ++cl) {
            if (cl > 0 && !(ok = W.wait(BAR(C::B_RD), (cl - 1) & 1))) break;
            tc_after();
#pragma unroll
            for (int i = 0; i < 4; ++i) tc_st16(tmem + lane_off + C::COL_AQ + 16 * i, pq + 16 * i);
            tc_wait_st();
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_AQF));
            if (cl > 0) {
                const int et = col_exp(p, cl - 1, cum);
                if constexpr (JAC)
                    q_drain_jac<DK, DV>(p, bh, nl, E, he.ek, he.ev, cl - 1, et, t, lane, tmem + lane_off, BAR(C::B_RF),
                                        sl);
                else
                    q_drain<DK, DV>(p, bh, part_base, nl, e_ms, E, he.ev, cl - 1, et, t, lane, tmem + lane_off,
                                    BAR(C::B_RF), qlp);
                if (p.colmax) cum += col_max(p, bh, cl - 1);
            }
#pragma unroll
            for (int s = 0; s < NL; ++s) qlp[s] = h_lo(xl[s]);
            {   // the next chunk's operand (its row is read after the drain, which needs the
                // registers; the load overlaps the readout now running).  Unconditional, so that
                // pq is provably dead during the drain (the last iteration builds an unused one).
                uint32_t x[C::XW];
                fetch_row<DK>(p.q16, p, bh, sl, cl + 1 < p.nc ? cl + 1 : cl, t, x, xl);
                p2q_dispatch<DK, 0, C::NPT>(ktile, x, pq);
            }
        }
        if (ok && p.nc > 0 && W.wait(BAR(C::B_RD), (p.nc - 1) & 1)) {
            const int et = col_exp(p, p.nc - 1, cum);
            if constexpr (JAC)
                q_drain_jac<DK, DV>(p, bh, nl, E, he.ek, he.ev, p.nc - 1, et, t, lane, tmem + lane_off, BAR(C::B_RF),
                                    sl);
            else
                q_drain<DK, DV>(p, bh, part_base, nl, e_ms, E, he.ev, p.nc - 1, et, t, lane, tmem + lane_off,
                                BAR(C::B_RF), qlp);
        }
        tc_before();
    } else {
        // ------------------------------------------------ state -> fp16 readout operand
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // pair row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t pw = p.pairs[ktile * 128 + r];
        const int ppair = ((int)(pw & 255u) < DK) + ((int)(pw >> 8) < DK);
        float cf[NL];
        int pe[NL], fi[NL], dg[NL];
#pragma unroll
        for (int s = 0; s < NL; ++s) {
            const int64_t at = ((int64_t)u * NL + s) * 128 + r;
            cf[s] = s < nl ? p.unit_coef[at] : 0.f;
            fi[s] = s < nl ? p.unit_fidx[at] : -1;
            dg[s] = ppair + (sl[s] < DK);               // degree of feature (pair r, l_s)
            // prefill: the feature's degree on both sides; gradient scan: the pair's degree on
            // both sides, the slot on the key side only
            pe[s] = JAC ? (dg[s] - 1) * E + he.ek : dg[s] * E;
            for (int i = 0; i < dg[s]; ++i) cf[s] *= p.inv_c;   // alpha_p = 1 / (p! c^p)
        }
        constexpr int NG = C::NG;
        const int ngu = NU / 16;
        const int ngv = nl * DV / 16;   // groups of V columns; group ngv holds the Z columns (and padding)
        float cum = 0.f;                // column maxima of the chunks before cl
        bool ok = true;
        if (p.load_state) {   // incoming state -> TMEM (prescaled frame)
            // a V group is 16 contiguous columns of one feature's S row (four 16-byte loads,
            // scaled by one factor); the Z group gathers one Z value per slot (each scaled
            // as it lands).  Two groups' loads are in flight before either is stored: each
            // group is a round trip to HBM, paid once per unit and segment.
            auto fetch = [&](int g, float4 (&x)[4], float &sc) {
                if (16 * g < nl * DV) {
                    const int sv = (16 * g) / DV;
                    const int f = seli(fi, sv);
                    sc = pow2f_sat(-(seli(dg, sv) * he.ek + he.ev));
                    const float4 *src = reinterpret_cast<const float4 *>(
                        p.S + (bh * p.F + (f >= 0 ? f : 0)) * (p.s_ld > 0 ? p.s_ld : DV) + p.s_off + (16 * g) % DV);
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[j] = f >= 0 ? src[j] : make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    sc = 1.f;
                    float z[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int sz = 16 * g + i - nl * DV;
                        z[i] = 0.f;
                        if (sz < nl) {
                            const int f = seli(fi, sz);
                            if (f >= 0) z[i] = p.Z[bh * p.F + f] * pow2f_sat(-(seli(dg, sz) * he.ek));
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[j] = make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
                }
            };
            auto put = [&](int g, const float4 (&x)[4], float sc) {
                uint32_t v16[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v16[4 * j] = __float_as_uint(x[j].x * sc);
                    v16[4 * j + 1] = __float_as_uint(x[j].y * sc);
                    v16[4 * j + 2] = __float_as_uint(x[j].z * sc);
                    v16[4 * j + 3] = __float_as_uint(x[j].w * sc);
                }
                tc_st16(tmem + lane_off + C::COL_S + 16 * g, v16);
            };
#pragma unroll 1
            for (int g = 0; g < ngu; g += 2) {
                float4 xa[4], xb[4];
                float sa = 1.f, sb = 1.f;
                fetch(g, xa, sa);
                if (g + 1 < ngu) fetch(g + 1, xb, sb);
                put(g, xa, sa);
                if (g + 1 < ngu) put(g + 1, xb, sb);
            }
            tc_wait_st();
        }
        for (int cl = 0; cl < p.nc && ok; ++cl) {
            const int b = cl & 1;
            if (cl > 0 && !(ok = W.wait(BAR(C::B_UD), (cl - 1) & 1))) break;
            // B double buffer: the readout of chunk cl-2 has read it
            if (cl >= 2 && !(ok = W.wait(BAR(C::B_BSE + b), ((cl >> 1) - 1) & 1))) break;
            tc_after();
            if (p.colmax && cl > 0) cum += col_max(p, bh, cl - 1);
            const int et = col_exp(p, cl, cum);
            const int sg = JAC ? jac_sigma(et, E, he.ek, p.P, p.lc) : state_sigma(et, e_ms, E, p.P, p.lc);
            float sc[NL];
#pragma unroll
            for (int s = 0; s < NL; ++s) sc[s] = cf[s] * pow2f_sat(pe[s] - sg);
            uint8_t *bs = smem + C::OFF_BS + b * C::W_BYTES + (r >> 3) * C::LBO + (r & 7) * 16;
            if (p.load_state || cl > 0) {
                // the V groups two at a time, the loads of the next pair in flight while this
                // pair converts; then the Z group, the last state read
                uint32_t ra[16], rb[16];
                tc_ld16(tmem + lane_off + C::COL_S, ra);
                if (1 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16, rb);
                tc_wait_ld();
#pragma unroll 1
                for (int g = 0; g < ngv; g += 2) {
                    uint32_t ha[8], hb[8];
                    conv_v(ra, sel(sc, (16 * g) / DV), ha);
                    if (g + 1 < ngv) conv_v(rb, sel(sc, (16 * g + 16) / DV), hb);
                    if (g + 2 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16 * (g + 2), ra);
                    if (g + 3 < ngv) tc_ld16(tmem + lane_off + C::COL_S + 16 * (g + 3), rb);
                    *reinterpret_cast<uint4 *>(bs + (2 * g) * 128) = make_uint4(ha[0], ha[1], ha[2], ha[3]);
                    *reinterpret_cast<uint4 *>(bs + (2 * g + 1) * 128) = make_uint4(ha[4], ha[5], ha[6], ha[7]);
                    if (g + 1 < ngv) {
                        *reinterpret_cast<uint4 *>(bs + (2 * g + 2) * 128) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                        *reinterpret_cast<uint4 *>(bs + (2 * g + 3) * 128) = make_uint4(hb[4], hb[5], hb[6], hb[7]);
                    }
                    if (g + 2 < ngv) tc_wait_ld();
                }
                tc_ld16(tmem + lane_off + C::COL_S + 16 * ngv, ra);
                tc_wait_ld();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_SR));   // state read: the update may proceed
                uint32_t hz[8];
                conv_z<NL>(ra, nl, sc, hz);
                *reinterpret_cast<uint4 *>(bs + (2 * ngv) * 128) = make_uint4(hz[0], hz[1], hz[2], hz[3]);
                *reinterpret_cast<uint4 *>(bs + (2 * ngv + 1) * 128) = make_uint4(hz[4], hz[5], hz[6], hz[7]);
            } else {   // fresh state before the first chunk: the operand is zero
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(C::B_SR));
#pragma unroll 1
                for (int g = 0; g < ngu; ++g) {
                    *reinterpret_cast<uint4 *>(bs + (2 * g) * 128) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(bs + (2 * g + 1) * 128) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::B_BSF + b));
        }
        if (ok && p.store_state && p.nc > 0 && W.wait(BAR(C::B_UD), (p.nc - 1) & 1)) {
            tc_after();
#pragma unroll 1
            for (int g = 0; g < NG; ++g) {
                if (g < ngu) {
                    uint32_t rr[16];
                    tc_ld16(tmem + lane_off + C::COL_S + 16 * g, rr);
                    tc_wait_ld();
                    if (16 * g < nl * DV) {   // 16 contiguous columns of one S row
                        const int sv = (16 * g) / DV;
                        const int f = seli(fi, sv);
                        const float sc = pow2f_sat(seli(dg, sv) * he.ek + he.ev);
                        if (f >= 0) {
                            float4 *dst = reinterpret_cast<float4 *>(p.S + (bh * p.F + f) * (p.s_ld > 0 ? p.s_ld : DV) +
                                                                     p.s_off + (16 * g) % DV);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                dst[j] = make_float4(__uint_as_float(rr[4 * j]) * sc, __uint_as_float(rr[4 * j + 1]) * sc,
                                                     __uint_as_float(rr[4 * j + 2]) * sc,
                                                     __uint_as_float(rr[4 * j + 3]) * sc);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int sz = 16 * g + i - nl * DV;
                            if (sz < nl) {
                                const int f = seli(fi, sz);
                                if (f >= 0)
                                    p.Z[bh * p.F + f] = __uint_as_float(rr[i]) * pow2f_sat(seli(dg, sz) * he.ek);
                            }
                        }
                    }
                }
            }
        }
        tc_before();
    }

    __syncthreads();
    if (warp == kWarpI) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

}  // namespace
}  // namespace sata
