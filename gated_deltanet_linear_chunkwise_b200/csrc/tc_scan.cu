// tc_scan.cu -- the scan over frames on the 5th-generation tensor cores.
//
// Carrying the state across frame f is the affine map Sig_{f+1} = M_f Sig_f + N_f
// (d_k x d_k and d_k x d_v per frame; the per-frame transition of the chunk = frame
// decomposition, and the pages' "prefix-sum composition of GDN transition
// matrices": cliffmar.tech article, "NVIDIA SANA-WM", training section on
// context parallelism).  The frames of one (b, h) chain are visited in order and
// the columns of the state evolve independently, so a few CTAs per chain, each
// owning up to 16 columns, keep the state on chip for the whole scan:
//   * the state lives in shared memory as the B operand of the next product,
//     split into bf16 hi + lo parts (hi = bf16(x), lo = bf16(x - hi));
//   * M_f arrives already split the same way (the transition kernel writes it in
//     the operand's 128-byte-swizzled K-major image) by one bulk copy one frame
//     ahead of its use (double buffer), prefetched into L2 two to four frames
//     ahead (the HBM latency stays off the serial chain);
//   * D = M_h Sig_h + M_h Sig_l + M_l Sig_h accumulates in fp32 in TMEM (the
//     dropped M_l Sig_l term is ~2^-16 relative), so the state keeps about
//     16 mantissa bits per step instead of bf16's 8;
//   * the epilogue (one thread per state row m) adds N_f (read into registers
//     while the products run), applies the chunk-reset rule, writes the bf16
//     state that the U and output kernels read, and writes the next operand.
// Warp roles (160 threads): warps 0-3 epilogue, warp 4 owns TMEM and one of its
// threads issues the bulk copies and the tcgen05.mma.  Every wait is bounded.
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kThreads = 160;
constexpr int kEpi = 128;

struct ScanGeom {
    int nslab_k, nslab_v;
    uint32_t mimg;      // bytes of one frame's M image (hi + lo)
    uint32_t sig_part;  // bytes of one part (hi or lo) of the state operand
    uint32_t pad;       // the products read 128 rows of every M slab: room past the last one
    uint32_t nstride;   // floats per staged row of N: d_v + 4, an odd number of 16-byte units,
                        // so the rows' float4 reads by consecutive threads hit distinct banks
    uint32_t sig_off, n_off, bar_off, total;
};

// Columns of the state one CTA carries: the columns of Sig evolve independently
// (Sig_{f+1}[:, c] = M_f Sig_f[:, c] + N_f[:, c]), so each chain's state is split over
// CTAs of at most 16 columns; each CTA streams the full M_f, and the chain's other CTAs
// find it in L2.
constexpr int kScanCols = 16;  // state columns per CTA (one 16-column TMEM chunk)
constexpr int kTmemCols = 32;  // the smallest TMEM allocation

__host__ __device__ inline ScanGeom scan_geom(int dk, int dv) {  // dv: the columns of one CTA
    ScanGeom g;
    g.nslab_k = (dk + 63) / 64;
    g.nslab_v = (dv + 63) / 64;
    g.mimg = 2u * g.nslab_k * dk * 128u;
    g.sig_part = (uint32_t)g.nslab_v * dk * 128u;
    g.pad = (uint32_t)(128 - dk) * 128u;
    g.sig_off = 2u * g.mimg;
    g.n_off = (g.sig_off + 2u * g.sig_part + g.pad + 15u) & ~15u;
    g.nstride = (uint32_t)dv + 4u;
    g.bar_off = g.n_off + (uint32_t)dk * g.nstride * 4u;
    g.total = g.bar_off + 64u;
    return g;
}

enum Bar { MFULL = 0, DFULL = 2, SREADY = 3, DRAIN = 4, NBAR = 5 };

// Element (row, col) of a 128-byte-swizzled image of 64-column slabs of `rows` rows:
// the K-major A image of M (row = m, col = l) and the MN-major B image of the state
// (row = l, the K index; col = c) share this layout.
__device__ __forceinline__ uint32_t img_off(int row, int col, int rows) {
    return sm100::sw128_kmajor_offset(row, col, rows);
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     sm100::smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
                 : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
k_scan_tc(const Problem p, const __nv_bfloat16 *__restrict__ Mimg, const float *__restrict__ Nb,
          __nv_bfloat16 *__restrict__ SigB, float *__restrict__ SigF, int *err, uint64_t wait_ns) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int dk = p.dk, ldv = p.dv;                  // ldv: the state's full column count (row stride)
    const int c_base = blockIdx.y * kScanCols;        // this CTA's columns [c_base, c_base + dv)
    const int dv = min(kScanCols, ldv - c_base);
    const ScanGeom geo = scan_geom(dk, dv);
    const long long chain = blockIdx.x;
    const long long F = p.F;
    const bool post = p.mode == GDN_MODE_FRAME;  // frame-wise: each frame's output state is the post-update one
    unsigned char *sM = smem;                         // 2 x M image
    unsigned char *sSh = smem + geo.sig_off;          // state hi (MN-major B image)
    unsigned char *sSl = sSh + geo.sig_part;          // state lo
    float *sN = (float *)(smem + geo.n_off);          // N_f, one row per epilogue thread
    uint64_t *bars = (uint64_t *)(smem + geo.bar_off);
    uint32_t *tmem_slot = (uint32_t *)(bars + NBAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (pass_failed(err)) return;  // an earlier stage of this pass gave up
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) sm100::mbar_init(&bars[i], i == SREADY ? kEpi : 1);
        sm100::fence_barrier_init();
    }
    if (warp == 4) {
        sm100::tmem_alloc(tmem_slot, kTmemCols);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t t_d = *tmem_slot;
    auto fh_of = [&](long long f) { return chain * F + scan_frame(p, f); };

    if (warp == 4) {
        // ------------------------------------------------------------ bulk copies + MMA issue
        if (lane == 0 && F > 0) {
            const uint32_t id = sm100::idesc_bf16(128, dv, 0, 1);
            const int nks = dk / 16;
            sm100::mbar_arrive_expect_tx(&bars[MFULL], geo.mimg);
            bulk_load(sM, Mimg + (size_t)fh_of(0) * (geo.mimg / 2), geo.mimg, &bars[MFULL]);
            long long issued = 1, waited = 0;  // frames whose M copy was issued / observed
            bool ok = true;
            long long f = 0;
            for (; f < F && ok; ++f) {
                const int buf = (int)(f & 1);
                // the state operand for frame f is in place once the epilogue of f - 1 (or the
                // initial load) has arrived; that also means the products of f - 1 are complete,
                // so the other M buffer is free for frame f + 1
                ok = sm100::mbar_wait(&bars[SREADY], (uint32_t)(f & 1), err, wait_ns);
                if (!ok) break;
                if (f + 1 < F) {
                    unsigned char *dst = sM + (buf ^ 1) * geo.mimg;
                    sm100::mbar_arrive_expect_tx(&bars[MFULL + (buf ^ 1)], geo.mimg);
                    bulk_load(dst, Mimg + (size_t)fh_of(f + 1) * (geo.mimg / 2), geo.mimg, &bars[MFULL + (buf ^ 1)]);
                    ++issued;
                }
                // the maps of the next frames into L2 ahead of their copies (HBM latency off the chain)
                for (int a = 2; a <= 4; ++a)
                    if (f + a < F) {
                        const long long fa = fh_of(f + a);
                        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Mimg + (size_t)fa * (geo.mimg / 2)),
                                     "r"(geo.mimg)
                                     : "memory");
                        if (blockIdx.y == 0)
                            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Nb + (size_t)fa * dk * ldv),
                                         "r"((uint32_t)(dk * ldv * 4))
                                         : "memory");
                    }
                ok = sm100::mbar_wait(&bars[MFULL + buf], (uint32_t)((f >> 1) & 1), err, wait_ns);
                if (!ok) break;
                ++waited;
                sm100::tc_fence_after();
                const unsigned char *mh = sM + buf * geo.mimg;
                const unsigned char *ml = mh + geo.mimg / 2;
                for (int ks = 0; ks < nks; ++ks)
                    sm100::mma_bf16_ss(t_d, desc_kmajor(mh, ks, dk), desc_mnmajor(sSh, ks, dk), id, ks > 0);
                for (int ks = 0; ks < nks; ++ks)
                    sm100::mma_bf16_ss(t_d, desc_kmajor(mh, ks, dk), desc_mnmajor(sSl, ks, dk), id, 1u);
                for (int ks = 0; ks < nks; ++ks)
                    sm100::mma_bf16_ss(t_d, desc_kmajor(ml, ks, dk), desc_mnmajor(sSh, ks, dk), id, 1u);
                sm100::mma_commit(&bars[DFULL]);
            }
            // leave with nothing in flight: every copy issued lands and every product issued
            // completes before TMEM and shared memory are released (full-limit drain waits)
            for (long long fr = waited; fr < issued; ++fr)
                sm100::mbar_wait(&bars[MFULL + (fr & 1)], (uint32_t)((fr >> 1) & 1), err, sm100::kWaitLimitNs, true);
            sm100::mma_commit(&bars[DRAIN]);
            sm100::mbar_wait(&bars[DRAIN], 0u, err, sm100::kWaitLimitNs, true);
        }
    } else {
        // ------------------------------------------------------------ epilogue: thread m owns state row m
        const int m = warp * 32 + lane;
        const bool row = m < dk;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float *sNrow = sN + m * geo.nstride;  // this thread's row of N_f (only this thread touches it)
        auto out_row = [&](long long f) -> long long { return (fh_of(f) * dk + m) * (long long)ldv + c_base; };
        // 16 columns [c0, c0 + 16) of a state row: the next product's operand (hi, lo) and
        // the bf16 / fp32 output rows
        auto put_operand = [&](const float (&x)[kScanCols], int c0) {
#pragma unroll
            for (int c8 = 0; c8 < kScanCols / 8; ++c8) {
                if (c0 + c8 * 8 >= dv) break;
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = x[c8 * 8 + 2 * e], b = x[c8 * 8 + 2 * e + 1];
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
                    const float2 hf = __bfloat1622float2(h2);
                    hi[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    lo[e] = pack_bf16(a - hf.x, b - hf.y);
                }
                const uint32_t off = img_off(m, c0 + c8 * 8, dk);
                *reinterpret_cast<uint4 *>(sSh + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sSl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        };
        auto put_out = [&](const float (&x)[kScanCols], int c0, long long f) {
            if (SigB) {
                __nv_bfloat16 *bd = SigB + out_row(f) + c0;
#pragma unroll
                for (int c8 = 0; c8 < kScanCols / 8; ++c8) {
                    if (c0 + c8 * 8 >= dv) break;
                    *reinterpret_cast<uint4 *>(bd + c8 * 8) = make_uint4(
                        pack_bf16(x[c8 * 8], x[c8 * 8 + 1]), pack_bf16(x[c8 * 8 + 2], x[c8 * 8 + 3]),
                        pack_bf16(x[c8 * 8 + 4], x[c8 * 8 + 5]), pack_bf16(x[c8 * 8 + 6], x[c8 * 8 + 7]));
                }
            }
            if (SigF) {
                float *fd = SigF + out_row(f) + c0;
#pragma unroll
                for (int c4 = 0; c4 < kScanCols / 4; ++c4) {
                    if (c0 + c4 * 4 >= dv) break;
                    *reinterpret_cast<float4 *>(fd + c4 * 4) =
                        make_float4(x[c4 * 4], x[c4 * 4 + 1], x[c4 * 4 + 2], x[c4 * 4 + 3]);
                }
            }
        };
        // ---- the initial state Sig_0 = S_in^T (or zero), the operand of frame 0's products
        if (row && F > 0) {
            for (int c0 = 0; c0 < dv; c0 += kScanCols) {
                float x[kScanCols];
#pragma unroll
                for (int e = 0; e < kScanCols; ++e)
                    x[e] = (p.S_in && c0 + e < dv) ? p.S_in[(chain * ldv + c_base + c0 + e) * (long long)dk + m] : 0.f;
                put_operand(x, c0);
                if (!post) put_out(x, c0, 0);  // token-wise: the state entering frame 0
            }
        }
        sm100::fence_proxy_async_smem();
        sm100::mbar_arrive(&bars[SREADY]);
        bool ok = true;
        for (long long f = 0; f < F && ok; ++f) {
            // N_f row m into shared memory while the products run
            if (row) {
                const float *src = Nb + (fh_of(f) * dk + m) * (long long)ldv + c_base;
                for (int c4 = 0; c4 < dv; c4 += 4) sm100::cp_async16(sNrow + c4, src + c4, 16);
            }
            sm100::cp_async_commit();
            ok = sm100::mbar_wait(&bars[DFULL], (uint32_t)(f & 1), err, wait_ns);
            sm100::cp_async_wait_all();
            if (!ok) break;
            sm100::tc_fence_after();
            const bool last = f + 1 == F;
            const bool reset_next = !last && frame_resets(p, f + 1);
            for (int c0 = 0; c0 < dv; c0 += kScanCols) {
                float x[kScanCols];
                sm100::tmem_ld16(t_d + lane_off + c0, x);
                sm100::tmem_ld_wait();
                if (!row) continue;
#pragma unroll
                for (int e = 0; e < kScanCols; e += 4) {
                    const float4 nn = *reinterpret_cast<const float4 *>(sNrow + c0 + e);
                    x[e] += nn.x;
                    x[e + 1] += nn.y;
                    x[e + 2] += nn.z;
                    x[e + 3] += nn.w;
                }
                if (post) put_out(x, c0, f);  // frame-wise: the frame's post-update state, before any reset
                if (!last) {
                    if (reset_next) {
#pragma unroll
                        for (int e = 0; e < kScanCols; ++e) x[e] = 0.f;
                    }
                    put_operand(x, c0);
                    if (!post) put_out(x, c0, f + 1);  // token-wise: the state entering frame f + 1
                } else if (p.S_out) {
#pragma unroll
                    for (int e = 0; e < kScanCols; ++e)
                        if (c0 + e < dv) p.S_out[(chain * ldv + c_base + c0 + e) * (long long)dk + m] = x[e];
                }
            }
            sm100::tc_fence_before();
            if (!last) {
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(&bars[SREADY]);
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(t_d, kTmemCols);
    }
}

}  // namespace

bool scan_tc_supported(int dk, int dv) {
    const ScanGeom g = scan_geom(dk, dv < kScanCols ? dv : kScanCols);
    return dk % 16 == 0 && dv % 16 == 0 && dk <= 128 && dv <= 128 && 1024 + g.total <= 227 * 1024;
}

size_t scan_mimg_bytes(int dk) {
    return (size_t)scan_geom(dk, 16).mimg;
}

cudaError_t launch_scan_tc(const Problem &p, const __nv_bfloat16 *Mimg, const float *Nb, __nv_bfloat16 *SigB,
                           float *SigF, int *err, uint64_t wait_ns, cudaStream_t s) {
    const ScanGeom g = scan_geom(p.dk, p.dv < kScanCols ? p.dv : kScanCols);
    const size_t smem = 1024 + g.total;
    cudaError_t e = cudaFuncSetAttribute(k_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.B * p.H), (unsigned)((p.dv + kScanCols - 1) / kScanCols));
    k_scan_tc<<<grid, kThreads, smem, s>>>(p, Mimg, Nb, SigB, SigF, err, wait_ns);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace gdn
