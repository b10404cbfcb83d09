// tc_u.cu -- pseudo-values U = Ub - W Sig on the tensor cores.
//
// With the state Sig entering a frame known, the frame's pseudo-values are
// U = Ub - W Sig (U = T (beta V - decayed K S) in the UT form of the delta
// rule; SANA-WM summary, "Memory-Efficient Long-Context Modeling
// (Section 3.2)", frame-wise GDN).  Persistent: one CTA per SM walks the
// 128-row blocks of its frame-heads: A = W (K-major, the last d_k columns of
// the [Ub | W] rows, through a 4-deep ring), B = Sig in bf16 (MN-major, the
// next frame-head's state loading into a second buffer), D = W Sig in a TMEM
// double buffer;
// the epilogue subtracts it from Ub and writes U in bf16, the B operand
// layout of the output kernel.
// The same kernel is the frame-wise operator's output (SANA-WM summary,
// "Memory-Efficient Long-Context Modeling (Section 3.2)", paragraph
// "Adaptation to video: frame-wise recurrence"): A = the frame's queries,
// Sig the state after the frame's update, and o = Q Sig written to o.
// Chunkwise, Ub arrives by tiled loads into a 2-deep ring, the epilogue forms
// U = Ub - W Sig in place there, and the producer stores the tile with U's
// tensor map: per-thread rows of Ub and U would touch 32 cache lines per warp
// access (rows 448 and 224 bytes apart).
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 192;
constexpr int NW = 3;  // ring depth of the W (or Q) tiles

struct Smem {
    static constexpr uint32_t SIG = 0;                     // 2 buffers x 2 slabs x d_k rows (<= 32 KB each)
    static constexpr uint32_t W = SIG + 4 * SLAB_BYTES;    // NW stages x 2 slabs x 128 rows
    static constexpr uint32_t UB = W + NW * 2 * SLAB_BYTES;  // 2 x (Ub, then U) tiles, chunkwise
    static constexpr uint32_t END = UB + 2 * 2 * SLAB_BYTES;
};
static_assert(1024 + Smem::END + 8 * 32 + 16 <= 232448, "over the 227 KB a CTA may use");

enum Bar {
    SIGFULL = 0, SIGEMPTY = 2, WFULL = 4, WEMPTY = WFULL + NW, QREADY = WEMPTY + NW, DFULL = QREADY + NW,
    DEMPTY = DFULL + 2, UBFULL = DEMPTY + 2, UREADY = UBFULL + 2, DRAIN = UREADY + 2, NBAR
};

// Persistent: one CTA per SM walks the 128-row blocks of its frame-heads (blockIdx.x +
// t gridDim.x); block i of the CTA's t-th frame-head is ring use g = t nblk + i, so the W
// tiles stream without a pause between frame-heads while the next state loads.
__global__ void __launch_bounds__(kThreads, 1)
k_u_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_q,
       const __grid_constant__ CUtensorMap tm_sig, const __grid_constant__ CUtensorMap tm_u, const UParams prm,
       long long n_fh) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int L = prm.L, dk = prm.dk, dv = prm.dv, nc = dk + dv, nblk = prm.nblk;
    unsigned char *sW = smem + Smem::W;
    uint64_t *bars = (uint64_t *)(smem + Smem::END);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int *err = prm.err;
    const uint64_t wait_ns = prm.wait_ns;
    const int nslab_k = (dk + SLAB - 1) / SLAB, nslab_v = (dv + SLAB - 1) / SLAB;
    const bool frame = prm.frame != 0;
    const bool normq = frame && prm.norm_q;
    const long long nmine = n_fh > blockIdx.x ? (n_fh - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const long long total = nmine * nblk;
    auto fh_of = [&](long long t) { return blockIdx.x + t * gridDim.x; };
    auto sig_buf = [&](long long t) { return smem + Smem::SIG + (t & 1) * 2 * SLAB_BYTES; };
    auto ub_buf = [&](long long g) { return smem + Smem::UB + (g & 1) * 2 * SLAB_BYTES; };

    if (pass_failed(prm.err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) {
            const bool many = (i >= QREADY && i < QREADY + NW) || i == DEMPTY || i == DEMPTY + 1 || i == UREADY ||
                              i == UREADY + 1;
            sm100::mbar_init(&bars[i], many ? 128 : 1);
        }
        sm100::fence_barrier_init();
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 256);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t t_d = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            sm100::tma_prefetch_desc(frame ? &tm_q : &tm_x);
            sm100::tma_prefetch_desc(&tm_sig);
            if (!frame) sm100::tma_prefetch_desc(&tm_u);
            // Streams, polled so that none waits on another's progress: each frame-head's state
            // ahead of its first block (once the products of frame-head t - 2 have read its
            // buffer), then W_g (the frame's Q) into the NW-deep ring once the product of use
            // g - NW has read the stage; chunkwise, U_g out of its Ub buffer once the epilogue has
            // formed it there, and Ub_g into buffer g & 1 once U_{g-2} has left it.
            long long gw = 0, tsig = 0;
            long long gu = frame ? total : 0, gs = frame ? total : 0;  // next Ub load, next U store
            bool ok = true;
            sm100::Spin spin(wait_ns);
            while (ok && (gw < total || gu < total || gs < total)) {
                bool prog = false;
                if (gw < total) {
                    const long long t = gw / nblk;
                    const int i = (int)(gw % nblk), st = (int)(gw % NW);
                    if (tsig <= t && tsig < nmine) {
                        if (tsig < 2 ||
                            sm100::mbar_test(&bars[SIGEMPTY + (tsig & 1)], (uint32_t)(((tsig >> 1) - 1) & 1))) {
                            sm100::mbar_arrive_expect_tx(&bars[SIGFULL + (tsig & 1)], (uint32_t)(nslab_v * dk * 128));
                            for (int sl = 0; sl < nslab_v; ++sl)
                                sm100::tma_load_3d(sig_buf(tsig) + sl * dk * 128, &tm_sig, &bars[SIGFULL + (tsig & 1)],
                                                   sl * SLAB, 0, (int)fh_of(tsig));
                            ++tsig;
                            prog = true;
                        }
                    } else if (gw < NW ||
                               sm100::mbar_test(&bars[WEMPTY + st], (uint32_t)(((gw / NW) - 1) & 1))) {
                        const long long fh = fh_of(t);
                        unsigned char *wst = sW + st * 2 * SLAB_BYTES;
                        sm100::mbar_arrive_expect_tx(&bars[WFULL + st], (uint32_t)(nslab_k * SLAB_BYTES));
                        for (int sl = 0; sl < nslab_k; ++sl) {
                            if (frame) {  // the frame's queries
                                const long long f = fh % prm.F, chain = fh / prm.F;
                                const int h = (int)(chain % prm.H), b = (int)(chain / prm.H);
                                sm100::tma_load_4d(wst + sl * SLAB_BYTES, &tm_q, &bars[WFULL + st], sl * SLAB, h,
                                                   i * BM, (int)(b * prm.F + f));
                            } else {  // W = columns dv .. dv + dk of the [Ub | W] rows
                                sm100::tma_load_3d(wst + sl * SLAB_BYTES, &tm_x, &bars[WFULL + st], dv + sl * SLAB,
                                                   i * BM, (int)fh);
                            }
                        }
                        ++gw;
                        prog = true;
                    }
                }
                if (gs < gu && sm100::mbar_test(&bars[UREADY + (gs & 1)], (uint32_t)((gs >> 1) & 1))) {
                    for (int sl = 0; sl < nslab_v; ++sl)
                        sm100::tma_store_3d(&tm_u, ub_buf(gs) + sl * SLAB_BYTES, sl * SLAB, (int)(gs % nblk) * BM,
                                            (int)fh_of(gs / nblk));
                    sm100::bulk_commit();
                    sm100::bulk_wait_read0();  // the buffer may take the next Ub once this returns
                    ++gs;
                    prog = true;
                }
                if (gu < total && gu < gs + 2) {  // columns 0 .. 127 of the [Ub | W] rows (Ub and a W margin)
                    sm100::mbar_arrive_expect_tx(&bars[UBFULL + (gu & 1)], (uint32_t)(nslab_v * SLAB_BYTES));
                    for (int sl = 0; sl < nslab_v; ++sl)
                        sm100::tma_load_3d(ub_buf(gu) + sl * SLAB_BYTES, &tm_x, &bars[UBFULL + (gu & 1)], sl * SLAB,
                                           (int)(gu % nblk) * BM, (int)fh_of(gu / nblk));
                    ++gu;
                    prog = true;
                }
                if (prog) {
                    spin.reset();
                } else if (!spin.tick(err)) {
                    ok = false;
                } else {
                    __nanosleep(64);
                }
            }
            // leave with no copy in flight (full-limit drain waits): the last NW tiles, the last two
            // Ub tiles and the states loaded for the last two frame-heads; the stores complete
            for (long long u = gw > NW ? gw - NW : 0; u < gw; ++u)
                sm100::mbar_wait(&bars[WFULL + (u % NW)], (uint32_t)((u / NW) & 1), err, sm100::kWaitLimitNs, true);
            if (!frame)
                for (long long u = gu > 2 ? gu - 2 : 0; u < gu; ++u)
                    sm100::mbar_wait(&bars[UBFULL + (u & 1)], (uint32_t)((u >> 1) & 1), err, sm100::kWaitLimitNs,
                                     true);
            for (long long u = tsig > 2 ? tsig - 2 : 0; u < tsig; ++u)
                sm100::mbar_wait(&bars[SIGFULL + (u & 1)], (uint32_t)((u >> 1) & 1), err, sm100::kWaitLimitNs, true);
            sm100::bulk_wait0();
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = sm100::idesc_bf16(BM, dv, 0, 1);
            bool ok = true;
            for (long long g = 0; g < total && ok; ++g) {
                const long long t = g / nblk;
                const int i = (int)(g % nblk), st = (int)(g % NW), db = (int)(g & 1);
                if (i == 0) ok = sm100::mbar_wait(&bars[SIGFULL + (t & 1)], (uint32_t)((t >> 1) & 1), err, wait_ns);
                // the operand is ready when it has landed, or (query feature map) once the
                // epilogue has normalised it in place
                if (ok) ok = sm100::mbar_wait(&bars[(normq ? QREADY : WFULL) + st], (uint32_t)((g / NW) & 1), err, wait_ns);
                if (ok && g >= 2) ok = sm100::mbar_wait(&bars[DEMPTY + db], (uint32_t)(((g >> 1) - 1) & 1), err, wait_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                const unsigned char *wt = sW + st * 2 * SLAB_BYTES;
                const unsigned char *sg = sig_buf(t);
                for (int ks = 0; ks < dk / 16; ++ks)
                    sm100::mma_bf16_ss(t_d + db * 128, desc_kmajor(wt, ks, BM), desc_mnmajor(sg, ks, dk), id,
                                       ks > 0);
                sm100::mma_commit(&bars[DFULL + db]);
                sm100::mma_commit(&bars[WEMPTY + st]);
                if (i == nblk - 1) sm100::mma_commit(&bars[SIGEMPTY + (t & 1)]);
            }
            sm100::mma_commit(&bars[DRAIN]);  // every product issued completes before TMEM is released
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        bool ok = true;
        // query feature map of the frame-wise operator (SANA-WM summary, section 3.2, "Algebraic
        // Stabilization for Spatial Token Explosion"): row r of use g's staged Q becomes
        // max(RMSNorm(q) w, 0) in place before the product reads it
        auto normalize = [&](long long g) -> bool {
            const int st = (int)(g % NW);
            if (!sm100::mbar_wait(&bars[WFULL + st], (uint32_t)((g / NW) & 1), err, wait_ns)) return false;
            unsigned char *wst = sW + st * 2 * SLAB_BYTES;
            float ss = 0.f;
            for (int sl = 0; sl < nslab_k; ++sl) {
                const uint4 *rowp = reinterpret_cast<const uint4 *>(wst + sl * SLAB_BYTES + r * 128);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint4 v = rowp[cc];
                    const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(p2[e]);
                        ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
                    }
                }
            }
            const float inv = 1.f / sqrtf(ss / (float)dk + kRmsEps);
            for (int sl = 0; sl < nslab_k; ++sl) {
                uint4 *rowp = reinterpret_cast<uint4 *>(wst + sl * SLAB_BYTES + r * 128);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 v = rowp[cc];
                    __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&v);
                    const int c0 = sl * 64 + ((cc ^ (r & 7)) << 3);  // logical column of the chunk
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(p2[e]);
                        const int ca = c0 + 2 * e;
                        const float wa = (prm.q_w && ca < dk) ? prm.q_w[ca] : 1.f;
                        const float wb = (prm.q_w && ca + 1 < dk) ? prm.q_w[ca + 1] : 1.f;
                        p2[e] = __floats2bfloat162_rn(fmaxf(x.x * inv * wa, 0.f), fmaxf(x.y * inv * wb, 0.f));
                    }
                    rowp[cc] = v;
                }
            }
            sm100::fence_proxy_async_smem();
            sm100::mbar_arrive(&bars[QREADY + st]);
            return true;
        };
        if (normq && total > 0) ok = normalize(0);
        for (long long g = 0; g < total && ok; ++g) {
            if (normq && g + 1 < total && !(ok = normalize(g + 1))) break;
            const long long t = g / nblk;
            const int i = (int)(g % nblk), db = (int)(g & 1);
            if (!frame) {  // U = Ub - D in place over use g's Ub tile; the producer stores it
                ok = sm100::mbar_wait(&bars[UBFULL + (g & 1)], (uint32_t)((g >> 1) & 1), err, wait_ns) &&
                     sm100::mbar_wait(&bars[DFULL + db], (uint32_t)((g >> 1) & 1), err, wait_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                unsigned char *ubt = ub_buf(g);
                tmem_walk16(t_d + db * 128 + lane_off, dv >> 4, [&](int j, const float (&d)[16]) {
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        uint4 *p = reinterpret_cast<uint4 *>(ubt + sw_offset(16 * j + 8 * w, r));
                        uint4 xv = *p;
                        __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&xv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 u = __bfloat1622float2(p2[e]);
                            p2[e] = __floats2bfloat162_rn(u.x - d[w * 8 + 2 * e], u.y - d[w * 8 + 2 * e + 1]);
                        }
                        *p = xv;
                    }
                });
                sm100::tc_fence_before();
                sm100::mbar_arrive(&bars[DEMPTY + db]);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[UREADY + (g & 1)]);
                continue;
            }
            const long long fh = fh_of(t);
            const long long f = frame ? fh % prm.F : 0, chain = frame ? fh / prm.F : 0;
            const int h = frame ? (int)(chain % prm.H) : 0, b = frame ? (int)(chain / prm.H) : 0;
            const int row = i * BM + r;
            const bool valid = row < L;
            // chunkwise: U = Ub - D over the row's [Ub | W]; frame-wise: o (+)= D
            const __nv_bfloat16 *xrow =
                frame ? prm.o + (((long long)b * prm.T + f * L + (valid ? row : 0)) * prm.H + h) * dv
                      : prm.X + (fh * (long long)L + (valid ? row : 0)) * nc;
            __nv_bfloat16 *urow = frame ? const_cast<__nv_bfloat16 *>(xrow)
                                        : prm.U + (fh * (long long)L + (valid ? row : 0)) * dv;
            const bool load_row = !frame || prm.accumulate;
            const float sgn = frame ? 1.f : -1.f;
            // this row's Ub (or the o being accumulated into) in registers before the wait, so
            // its latency hides behind the MMA
            uint4 ub[16];
#pragma unroll
            for (int c8 = 0; c8 < 16; ++c8)
                ub[c8] = (valid && load_row && c8 < dv / 8) ? __ldg(reinterpret_cast<const uint4 *>(xrow) + c8)
                                                            : make_uint4(0, 0, 0, 0);
            ok = sm100::mbar_wait(&bars[DFULL + db], (uint32_t)((g >> 1) & 1), err, wait_ns);
            if (!ok) break;
            sm100::tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c0 = 16 * j;
                if (c0 >= dv) break;
                float d[16];
                sm100::tmem_ld16(t_d + db * 128 + lane_off + c0, d);
                sm100::tmem_ld_wait();
                if (valid) {
                    uint4 out[2];
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        uint4 xv = ub[2 * j + w];
                        __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&xv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 u = __bfloat1622float2(p2[e]);
                            p2[e] = __floats2bfloat162_rn(u.x + sgn * d[w * 8 + 2 * e], u.y + sgn * d[w * 8 + 2 * e + 1]);
                        }
                        out[w] = xv;
                    }
                    reinterpret_cast<uint4 *>(urow + c0)[0] = out[0];
                    reinterpret_cast<uint4 *>(urow + c0)[1] = out[1];
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(&bars[DEMPTY + db]);
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(t_d, 256);
    }
}

}  // namespace

cudaError_t launch_u_tc(const CUtensorMap &tm_x, const CUtensorMap &tm_q, const CUtensorMap &tm_sig,
                        const CUtensorMap &tm_u, const UParams &prm, long long n_fh, int num_sms, cudaStream_t s) {
    const size_t smem = 1024 + Smem::END + sizeof(uint64_t) * NBAR + 16;
    cudaError_t e = cudaFuncSetAttribute(k_u_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = n_fh < num_sms ? n_fh : num_sms;
    if (grid <= 0) return cudaSuccess;
    k_u_tc<<<(unsigned)grid, kThreads, smem, s>>>(tm_x, tm_q, tm_sig, tm_u, prm, n_fh);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
