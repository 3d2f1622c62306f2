// scan_fwd.cu -- S6 selective-scan forward engine.
//
// Arithmetic ("vision mamba-yolov8", section "2. Vmamba module code",
// selective_scan_ref): dt = softplus(delta + bias); per state n
// h = exp(dt*A[c,n]) * h + dt*B[n,l]*u; y = sum_n C[n,l]*h + D[c]*u; h = 0 at
// the start; channel c = k*D + d uses the B/C group k.
//
// Design (B200, sm_100a).  The work is one exponential per state update, so
// the engine is bound by the SFU (MUFU.EX2: 16 per clock per SM) and by issue
// slots, not by HBM.  Each thread owns one whole (b, c) sequence with all N
// states in registers and walks it in order: per state update that is one
// FMUL (dt * A*log2e), one MUFU.EX2, one FMUL (dt*u * B) and two FFMAs -- no
// cross-thread scan arithmetic at all.
//
//  * A CTA is one warp: 32 channels of one (b, k), 16 warps resident per SM
//    (four per scheduler).
//  * B[., l] and C[., l] are the same for all 32 threads (group k of batch b);
//    each thread's u and delta rows are its own.  All of them are staged in
//    shared memory in 8-step chunks with cp.async (16-byte pieces for fp32,
//    8-byte for bf16), double buffered, and read as 4-step vector loads.
//  * The fused SS2D forward reads u from the image along path k: row-major
//    paths from x (k=2 backwards), column-major paths from a transposed copy
//    of x (k=3 backwards), so every load stays sequential.
//  * The bidirectional scan (bimamba_inner_ref) runs a sequence and its reverse
//    as two directions of one launch; the reverse direction stages x, delta, B
//    and C backwards (4-step pieces copied in memory order, read from the end)
//    and stores its outputs at their natural positions.
//
// When a problem has too few sequences to fill the GPU, each sequence is cut
// into segments: a summary pass computes, per segment, the state reached
// from zero and the decay product exp(A * sum dt); the output pass starts
// each segment from the carry combined over the segments before it.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kWarp = 32;   // threads (= channels) per CTA
// steps staged per chunk (B/C, u, delta); shorter chunks use less shared memory per CTA
#ifndef SS2D_FWD_LC
#define SS2D_FWD_LC 8
#endif
constexpr int kLC = SS2D_FWD_LC;
constexpr int kG = 4;       // steps per register group
constexpr int kStateChunk = SS2D_CHUNK_LEN;

// Resident CTAs (warps) per SM the forward kernel is compiled for.  16 keeps four
// warps on each of the SM's four schedulers (13 or 21 would leave one scheduler a
// warp more than the others) and leaves 128 registers per lane, enough for the
// unrolled 16-state loop without spills; fewer registers (e.g. 96 for 20 warps)
// spill and measured slower.
#ifndef SS2D_FWD_MIN_BLOCKS
#define SS2D_FWD_MIN_BLOCKS 16
#endif
// Of every 16 states, how many take their exponentials from the FMA-pipe
// polynomial (ex2_poly2) instead of the SFU, to balance the two pipes.
#ifndef SS2D_FWD_POLY_STATES
#define SS2D_FWD_POLY_STATES 0
#endif
// 1: the y readout sums even and odd states in two accumulators (shorter chains)
#ifndef SS2D_FWD_YSPLIT
#define SS2D_FWD_YSPLIT 0
#endif
// 1: A*log2(e) per (lane, state) lives in shared memory (fewer registers);
// 0: in registers for fp32 inputs (fewer shared-memory loads), shared memory for bf16
#ifndef SS2D_FWD_A2_SMEM
#define SS2D_FWD_A2_SMEM 0
#endif

struct FwdParams {
    const void *u;       // (B, 4D, L) sequences, or image x (B, D, H, W)
    const void *uT;      // transposed image (B, D, W, H) for the column paths (image mode)
    const void *delta;
    const float *A;
    const void *Bm;
    const void *Cm;
    const float *Dv;
    const float *bias;
    void *out;
    float *chunk_states;
    const void *z;       // (B, 4D, L) output gate or null (sequence mode only)
    float *last_state;   // (B, 4D, N) or null
    float *seg;  // (B, 4D, nseg, 2, N): decay product and end state of each segment
    const void *xdbl;    // projection mode: (B, 4, R+2N, L) per-path x_proj outputs, in_dtype
    const float *Wdt;    // projection mode: (4D, R)
    int R;
    int64_t B, D, H, W, L;
    int N;
    int softplus;
    int nseg;
    int64_t seglen;
    int64_t nchunks;
};

template <typename T>
__device__ __forceinline__ void cp_async_bytes(T *smem_dst, const T *gsrc, int bytes) {
    const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(gsrc));
    else if (bytes == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(gsrc));
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(gsrc));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Shared-memory staging of one chunk (kLC steps):
//  * B/C of group (b, k): [NS][kLC], shared by the 32 lanes;
//  * each lane's u and delta rows: [32][kRow], rows padded to kRow elements so
//    the per-lane 4-step vector reads hit distinct banks.  A reversed u row
//    (paths 2, 3) is copied in memory order: step cbeg+i sits at kLC-1-i.
template <typename Tin, int NS>
struct FwdStage {
    static constexpr int kRow = kLC + 4;
    Tin B[NS][kLC];
    Tin C[NS][kLC];
    Tin U[kWarp][kRow];
    Tin Dl[kWarp][kRow];
};

// Shared-memory slots are the same in every form: slot i of a row holds step cbeg+i,
// or step cbeg+kLC-1-i for a reversed row, so the scan reads 4-step vectors.
// Issue the copies of chunk [cbeg, cbeg+len):
//  * VEC (rows 16-byte aligned, len a multiple of 4): 4-element cp.async pieces;
//  * fp32 rows of any alignment: one 4-byte cp.async per element, slots past the end zeroed;
//  * bf16 rows of any alignment: plain loads (synchronous), slots past the end zeroed.
// REV: the chunk is walked backwards through delta, B and C as well (bidirectional scan).
// PROJ: instead of each lane's delta row, the R <= RB low-rank dt rows of the group (dts, like B/C).
template <int NS, bool VEC, bool REV, bool PROJ, int RB, typename Tin>
__device__ __forceinline__ void stage_chunk(FwdStage<Tin, NS> &st, const Tin *Bk, const Tin *Ck, int N, int64_t L,
                                            const Tin *urow, bool urev, const Tin *drow, bool active, int64_t cbeg,
                                            int len, Tin (*dts)[kLC] = nullptr, const Tin *DTk = nullptr,
                                            int R = 0) {
    const int t = threadIdx.x;
    constexpr int kBytes = 4 * (int)sizeof(Tin);
    if (PROJ) {  // the group's dt rows, in the same slots as B/C
        for (int idx = t; idx < RB * kLC; idx += kWarp) {
            const int r = idx / kLC, i = idx % kLC;
            if (VEC) {
                if (i % 4 == 0 && r < R && i < len)
                    cp_async_bytes(&dts[r][i], DTk + (int64_t)r * L + cbeg + i, kBytes);
            } else if (sizeof(Tin) == 4) {
                if (r < R && i < len)
                    cp_async_bytes(&dts[r][i], DTk + (int64_t)r * L + cbeg + i, 4);
                else
                    dts[r][i] = Tin(0.f);
            } else {
                dts[r][i] = (r < R && i < len) ? DTk[(int64_t)r * L + cbeg + i] : Tin(0.f);
            }
        }
    }
    if (VEC) {
        constexpr int q = kLC / 4;
        for (int idx = t; idx < NS * q; idx += kWarp) {
            const int n = idx / q, i4 = (idx % q) * 4;
            if (n < N && i4 < len) {
                if (!REV) {
                    cp_async_bytes(&st.B[n][i4], Bk + (int64_t)n * L + cbeg + i4, kBytes);
                    cp_async_bytes(&st.C[n][i4], Ck + (int64_t)n * L + cbeg + i4, kBytes);
                } else {
                    cp_async_bytes(&st.B[n][kLC - 4 - i4], Bk + (int64_t)n * L + (L - cbeg - 4 - i4), kBytes);
                    cp_async_bytes(&st.C[n][kLC - 4 - i4], Ck + (int64_t)n * L + (L - cbeg - 4 - i4), kBytes);
                }
            }
        }
        if (active) {
#pragma unroll
            for (int i4 = 0; i4 < kLC; i4 += 4) {
                if (i4 < len) {
                    if (PROJ)
                        ;  // no delta row: dt comes from the projection
                    else if (!REV)
                        cp_async_bytes(&st.Dl[t][i4], drow + cbeg + i4, kBytes);
                    else
                        cp_async_bytes(&st.Dl[t][kLC - 4 - i4], drow + (L - cbeg - 4 - i4), kBytes);
                    if (!urev)
                        cp_async_bytes(&st.U[t][i4], urow + cbeg + i4, kBytes);
                    else  // steps cbeg+i4 .. +3 live at memory L-1-cbeg-i4-3 .. L-1-cbeg-i4
                        cp_async_bytes(&st.U[t][kLC - 4 - i4], urow + (L - cbeg - 4 - i4), kBytes);
                }
            }
        }
    } else if (sizeof(Tin) == 4) {
        for (int idx = t; idx < NS * kLC; idx += kWarp) {
            const int n = idx / kLC, i = idx % kLC;
            const int slot = REV ? kLC - 1 - i : i;
            if (n < N && i < len) {
                const int64_t m = REV ? L - 1 - (cbeg + i) : cbeg + i;
                cp_async_bytes(&st.B[n][slot], Bk + (int64_t)n * L + m, 4);
                cp_async_bytes(&st.C[n][slot], Ck + (int64_t)n * L + m, 4);
            } else {
                st.B[n][slot] = Tin(0.f);
                st.C[n][slot] = Tin(0.f);
            }
        }
        for (int i = 0; i < kLC; ++i) {
            const int64_t l = cbeg + i;
            const int dslot = REV ? kLC - 1 - i : i, uslot = urev ? kLC - 1 - i : i;
            if (active && i < len) {
                if (!PROJ) cp_async_bytes(&st.Dl[t][dslot], drow + (REV ? L - 1 - l : l), 4);
                cp_async_bytes(&st.U[t][uslot], urow + (urev ? L - 1 - l : l), 4);
            } else {
                st.Dl[t][dslot] = Tin(0.f);
                st.U[t][uslot] = Tin(0.f);
            }
        }
    } else {
        for (int idx = t; idx < NS * kLC; idx += kWarp) {
            const int n = idx / kLC, i = idx % kLC;
            const bool ok = n < N && i < len;
            const int64_t m = REV ? L - 1 - (cbeg + i) : cbeg + i;
            const int slot = REV ? kLC - 1 - i : i;
            st.B[n][slot] = ok ? Bk[(int64_t)n * L + m] : Tin(0.f);
            st.C[n][slot] = ok ? Ck[(int64_t)n * L + m] : Tin(0.f);
        }
        for (int i = 0; i < kLC; ++i) {
            const bool ok = active && i < len;
            const int64_t l = cbeg + i;
            if (!PROJ) st.Dl[t][REV ? kLC - 1 - i : i] = ok ? drow[REV ? L - 1 - l : l] : Tin(0.f);
            st.U[t][urev ? (kLC - 1 - i) : i] = ok ? urow[urev ? (L - 1 - l) : l] : Tin(0.f);
        }
    }
}

// A[c, n] * log2(e) of each lane's channel: in registers for fp32 inputs, in shared memory
// for bf16 (whose conversions need the registers)
template <typename Tin>
__host__ __device__ constexpr bool a2_in_smem() {
    return SS2D_FWD_A2_SMEM || sizeof(Tin) < 4;
}

// The scan of one CTA.  PASS 0: single pass.  PASS 1: segment summaries only.  PASS 2:
// outputs with carries.  REV: the reverse direction of the bidirectional scan.
// dt ranks the projection modes' shared arrays are sized for
template <int MODE>
__host__ __device__ constexpr int proj_rank_bucket() {
    return MODE == kModeImgProj ? kProjRNarrow : 1;
}

template <int NS, typename Tin, typename Tout, int MODE, int PASS, bool VEC, bool REV>
__device__ __forceinline__ void scan_fwd_body(const FwdParams &p, FwdStage<Tin, NS> (&stage)[2],
                                              float (&A2s)[a2_in_smem<Tin>() ? NS : 1][kWarp],
                                              Tin (*dts)[proj_rank_bucket<MODE>()][kLC], float (*wsm)[kWarp]) {
    constexpr bool PROJ = MODE == kModeImgProj || MODE == kModeImgProjWide;  // B, C from x_dbl
    constexpr bool DTIN = MODE == kModeImgProj;  // dt projected here, not read from delta
    constexpr int RB = proj_rank_bucket<MODE>();
    constexpr bool IMG = MODE == kModeImg || PROJ, BIDIR = MODE == kModeBidir, SEQ = MODE == kModeSeq;
    constexpr bool kA2Smem = a2_in_smem<Tin>();
    float A2r[NS];
#define SS2D_A2(n) (kA2Smem ? A2s[n][t] : A2r[n])

    const int t = threadIdx.x;
    const int k = blockIdx.y;
    const int64_t b = blockIdx.z / p.nseg;
    const int sgi = blockIdx.z % p.nseg;
    const int64_t D = p.D, L = p.L, C4 = (BIDIR ? 2 : kPaths) * p.D;
    const int64_t d = (int64_t)blockIdx.x * kWarp + t;
    const bool active = d < D;
    const int64_t c = k * D + (active ? d : 0);
    const int N = p.N;
    const int64_t lbeg = (int64_t)sgi * p.seglen;
    const int64_t lend = min(L, lbeg + p.seglen);

    float h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        const float a2v = (active && n < N) ? p.A[c * N + n] * kLog2e : 0.f;
        if (kA2Smem)
            A2s[n][t] = a2v;
        else
            A2r[n] = a2v;
        h[n] = 0.f;
    }
    if (DTIN) {  // this lane's row of dt_proj, kept in shared memory (lanes fastest)
#pragma unroll
        for (int r = 0; r < RB; ++r) wsm[r][t] = (active && r < p.R) ? p.Wdt[c * p.R + r] : 0.f;
    }
    const int64_t pc = BIDIR ? (active ? d : 0) : c;  // D and delta_bias are shared by the two directions
    const float Dc = (active && p.Dv) ? p.Dv[pc] : 0.f;
    const float bias = (active && p.bias) ? p.bias[pc] : 0.f;
    if (PASS == 2 && active) {
        // carry into this segment: fold the summaries of the segments before it
        const float *sg = p.seg + (b * C4 + c) * (int64_t)p.nseg * 2 * N;
        for (int s2 = 0; s2 < sgi; ++s2) {
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N) h[n] = fmaf(sg[(s2 * 2 + 0) * N + n], h[n], sg[(s2 * 2 + 1) * N + n]);
        }
    }
    float dtsum = 0.f;

    // this lane's u and delta sequences
    const Tin *urow;
    bool urev;
    if (IMG) {
        const Tin *img = static_cast<const Tin *>((k & 1) ? p.uT : p.u);
        urow = img + (b * D + (active ? d : 0)) * L;
        urev = k >= 2;
    } else if (BIDIR) {
        urow = static_cast<const Tin *>(p.u) + (b * D + (active ? d : 0)) * L;
        urev = REV;
    } else {
        urow = static_cast<const Tin *>(p.u) + (b * C4 + c) * L;
        urev = false;
    }
    const Tin *drow =
        DTIN ? nullptr : static_cast<const Tin *>(p.delta) + (BIDIR ? b * D + (active ? d : 0) : b * C4 + c) * L;
    const int64_t grp = BIDIR ? b : b * kPaths + k;  // the B/C group of this (b, k)
    // projection mode: the group's x_proj outputs are R dt rows, then N rows of B, then N of C
    const Tin *DTk = PROJ ? static_cast<const Tin *>(p.xdbl) + grp * (p.R + 2 * N) * L : nullptr;
    const Tin *Bk = PROJ ? DTk + (int64_t)p.R * L : static_cast<const Tin *>(p.Bm) + grp * N * L;
    const Tin *Ck = PROJ ? Bk + (int64_t)N * L : static_cast<const Tin *>(p.Cm) + grp * N * L;
    Tout *orow = p.out ? static_cast<Tout *>(p.out) + (b * C4 + c) * L : nullptr;

    const int64_t nloc = lend - lbeg;
    const int nchunk = (int)ceil_div(nloc, kLC);

    // rows n >= N of the B/C buffers are never copied: zero them once so padded
    // states stay at h = 0 and contribute nothing
    if (VEC && N < NS) {
        for (int sb = 0; sb < 2; ++sb)
            for (int i = t; i < NS * kLC; i += kWarp) {
                (&stage[sb].B[0][0])[i] = Tin(0.f);
                (&stage[sb].C[0][0])[i] = Tin(0.f);
            }
    }
    __syncwarp();

    stage_chunk<NS, VEC, REV, DTIN, RB>(stage[0], Bk, Ck, N, L, urow, urev, drow, active, lbeg,
                                    (int)min((int64_t)kLC, nloc), DTIN ? dts[0] : nullptr, DTk, p.R);
    cp_async_commit();

    for (int ch = 0; ch < nchunk; ++ch) {
        const int64_t cbeg = lbeg + (int64_t)ch * kLC;
        const int clen = (int)min((int64_t)kLC, lend - cbeg);
        const int buf = ch & 1;
        if (ch + 1 < nchunk) {
            const int64_t nbeg = cbeg + kLC;
            stage_chunk<NS, VEC, REV, DTIN, RB>(stage[buf ^ 1], Bk, Ck, N, L, urow, urev, drow, active, nbeg,
                                            (int)min((int64_t)kLC, lend - nbeg), DTIN ? dts[buf ^ 1] : nullptr, DTk,
                                            p.R);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const FwdStage<Tin, NS> &sm = stage[buf];

        if (active) {
            for (int g = 0; g < clen; g += kG) {
                const int64_t l0 = cbeg + g;
                const int nvalid = (int)min((int64_t)kG, lend - l0);
                float uv[kG], dv[kG];
                {  // slots hold 4-step groups in every staging form (see stage_chunk)
                    if (DTIN) {  // delta = dt_proj . x_dbl[:R] for the four steps
                        float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int r = 0; r < RB; ++r) {
                            if (r < p.R) {
                                const float w = wsm[r][t];
                                float q[kG];
                                ld4(&dts[buf][r][g], q);
                                a01 = __ffma2_rn(make_float2(w, w), make_float2(q[0], q[1]), a01);
                                a23 = __ffma2_rn(make_float2(w, w), make_float2(q[2], q[3]), a23);
                            }
                        }
                        dv[0] = a01.x;
                        dv[1] = a01.y;
                        dv[2] = a23.x;
                        dv[3] = a23.y;
                    } else if (!REV) {
                        ld4(&sm.Dl[t][g], dv);
                    } else {
                        float w[kG];
                        ld4(&sm.Dl[t][kLC - 4 - g], w);
                        dv[0] = w[3];
                        dv[1] = w[2];
                        dv[2] = w[1];
                        dv[3] = w[0];
                    }
                    if (!urev) {
                        ld4(&sm.U[t][g], uv);
                    } else {
                        float w[kG];
                        ld4(&sm.U[t][kLC - 4 - g], w);
                        uv[0] = w[3];
                        uv[1] = w[2];
                        uv[2] = w[1];
                        uv[3] = w[0];
                    }
                }
                // step pairs (0,1) and (2,3) ride the packed fp32 pipe (f32x2)
                const float2 t01 = make_float2(dv[0] + bias, dv[1] + bias);
                const float2 t23 = make_float2(dv[2] + bias, dv[3] + bias);
                float2 dt01 = p.softplus ? softplus_f2(t01) : t01;
                float2 dt23 = p.softplus ? softplus_f2(t23) : t23;
                if (!VEC && nvalid < kG) {
                    // steps past the end keep h unchanged: dt = 0 gives decay 1 and input 0
                    if (nvalid < 2) dt01.y = 0.f;
                    if (nvalid < 3) dt23.x = 0.f;
                    dt23.y = 0.f;
                }
                const float2 u01 = make_float2(uv[0], uv[1]), u23 = make_float2(uv[2], uv[3]);
                const float2 dtu01 = __fmul2_rn(dt01, u01), dtu23 = __fmul2_rn(dt23, u23);
                // skip term first: u is not needed during the state loop.  Even and odd
                // states accumulate separately, halving the dependent chain of adds.
                float2 y01 = __fmul2_rn(make_float2(Dc, Dc), u01);
                float2 y23 = __fmul2_rn(make_float2(Dc, Dc), u23);
                float2 z01 = make_float2(0.f, 0.f), z23 = make_float2(0.f, 0.f);
#pragma unroll
                for (int n = 0; n < NS; ++n) {
                    const float a2s = SS2D_A2(n);
                    const float2 a2 = make_float2(a2s, a2s);
                    float bq[kG], cq[kG];
                    if (!REV) {
                        ld4(&sm.B[n][g], bq);
                        ld4(&sm.C[n][g], cq);
                    } else {
                        float wb[kG], wc[kG];
                        ld4(&sm.B[n][kLC - 4 - g], wb);
                        ld4(&sm.C[n][kLC - 4 - g], wc);
#pragma unroll
                        for (int j = 0; j < kG; ++j) {
                            bq[j] = wb[kG - 1 - j];
                            cq[j] = wc[kG - 1 - j];
                        }
                    }
                    const float2 x01 = __fmul2_rn(dt01, a2), x23 = __fmul2_rn(dt23, a2);
                    const float2 b01 = __fmul2_rn(dtu01, make_float2(bq[0], bq[1]));
                    const float2 b23 = __fmul2_rn(dtu23, make_float2(bq[2], bq[3]));
                    float2 e01, e23;
                    if (n >= NS - (SS2D_FWD_POLY_STATES * NS) / 16) {  // FMA-pipe exponentials
                        e01 = ex2_poly2(x01);
                        e23 = ex2_poly2(x23);
                    } else {
                        e01 = make_float2(ex2_sfu(x01.x), ex2_sfu(x01.y));
                        e23 = make_float2(ex2_sfu(x23.x), ex2_sfu(x23.y));
                    }
                    const float h0 = fmaf(e01.x, h[n], b01.x);
                    const float h1 = fmaf(e01.y, h0, b01.y);
                    const float h2 = fmaf(e23.x, h1, b23.x);
                    const float h3 = fmaf(e23.y, h2, b23.y);
                    h[n] = h3;
                    if (SS2D_FWD_YSPLIT && (n & 1)) {
                        z01 = __ffma2_rn(make_float2(cq[0], cq[1]), make_float2(h0, h1), z01);
                        z23 = __ffma2_rn(make_float2(cq[2], cq[3]), make_float2(h2, h3), z23);
                    } else {
                        y01 = __ffma2_rn(make_float2(cq[0], cq[1]), make_float2(h0, h1), y01);
                        y23 = __ffma2_rn(make_float2(cq[2], cq[3]), make_float2(h2, h3), y23);
                    }
                }
                if (SS2D_FWD_YSPLIT) {
                    y01 = __fadd2_rn(y01, z01);
                    y23 = __fadd2_rn(y23, z23);
                }
                if (PASS == 1) {
                    dtsum += (dt01.x + dt01.y) + (dt23.x + dt23.y);
                } else {
                    float y[kG] = {y01.x, y01.y, y23.x, y23.y};
                    if (SEQ && p.z) {  // output gate: y * silu(z), after the D u term
                        const Tin *zrow = static_cast<const Tin *>(p.z) + (b * C4 + c) * L;
                        float zv[kG];
                        if (VEC) {
                            ld4(zrow + l0, zv);
                        } else {
#pragma unroll
                            for (int j = 0; j < kG; ++j) zv[j] = j < nvalid ? ld(zrow + l0 + j) : 0.f;
                        }
#pragma unroll
                        for (int j = 0; j < kG; ++j) y[j] *= silu_f(zv[j]);
                    }
                    if (orow) {
                        if (VEC && !REV) {
                            st4(orow + l0, y);
                        } else if (VEC) {  // the reverse direction stores at the natural positions
                            const float yr[kG] = {y[3], y[2], y[1], y[0]};
                            st4(orow + (L - kG - l0), yr);
                        } else {
#pragma unroll
                            for (int j = 0; j < kG; ++j)
                                if (j < nvalid) st(orow + (REV ? L - 1 - (l0 + j) : l0 + j), y[j]);
                        }
                    }
                    const int64_t llast = l0 + nvalid - 1;
                    if (p.chunk_states && (((llast + 1) % kStateChunk) == 0 || llast + 1 == L)) {
                        float *cs = p.chunk_states + ((b * C4 + c) * p.nchunks + llast / kStateChunk) * N;
                        if (N == NS && NS % 4 == 0) {  // 16-byte aligned rows of N floats
#pragma unroll
                            for (int n = 0; n < NS; n += 4) st4(cs + n, &h[n]);
                        } else {
#pragma unroll
                            for (int n = 0; n < NS; ++n)
                                if (n < N) cs[n] = h[n];
                        }
                    }
                }
            }
        }
        __syncwarp();  // every lane is done with this buffer before it is refilled
    }

    if (SEQ && PASS != 1 && active && p.last_state && sgi == p.nseg - 1) {  // sequence mode only
        float *ls = p.last_state + (b * C4 + c) * N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < N) ls[n] = h[n];
    }
    if (PASS == 1 && active) {
        float *sg = p.seg + ((b * C4 + c) * (int64_t)p.nseg + sgi) * 2 * N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < N) {
                sg[n] = ex2_sfu(SS2D_A2(n) * dtsum);
                sg[N + n] = h[n];
            }
    }
}

#undef SS2D_A2

template <int NS, typename Tin, typename Tout, int MODE, int PASS, bool VEC>
__global__ void __launch_bounds__(kWarp, SS2D_FWD_MIN_BLOCKS) scan_fwd_kernel(const FwdParams p) {
    __shared__ __align__(16) FwdStage<Tin, NS> stage[2];
    __shared__ float A2s[a2_in_smem<Tin>() ? NS : 1][kWarp];
    if constexpr (MODE == kModeImgProj) {  // dt rows, each lane's dt_proj row
        __shared__ __align__(16) Tin dts[2][proj_rank_bucket<MODE>()][kLC];
        __shared__ float wsm[proj_rank_bucket<MODE>()][kWarp];
        scan_fwd_body<NS, Tin, Tout, MODE, PASS, VEC, false>(p, stage, A2s, dts, wsm);
    } else if (MODE == kModeBidir && blockIdx.y == 1) {
        scan_fwd_body<NS, Tin, Tout, MODE, PASS, VEC, true>(p, stage, A2s, nullptr, nullptr);
    } else {
        scan_fwd_body<NS, Tin, Tout, MODE, PASS, VEC, false>(p, stage, A2s, nullptr, nullptr);
    }
}

// Segment plan: how many segments each sequence is cut into, and their length
// (a multiple of the state-chunk length).  One segment means a single pass.
static void seg_plan(const LaunchShape &s, int paths, int max_segments, int *nseg_out, int64_t *seglen_out) {
    // aim for at least ~512 resident sequences (threads) per SM on 148 SMs
    const int64_t seqs = s.B * paths * s.D;
    const int64_t target = 148LL * 512;
    *nseg_out = 1;
    *seglen_out = s.L;
    if (seqs >= target || s.L <= 2 * kStateChunk) return;
    int64_t nseg = ceil_div(target, seqs);
    const int64_t max_seg = ceil_div(s.L, kStateChunk);
    if (nseg > max_seg) nseg = max_seg;
    if (nseg > max_segments) nseg = max_segments;
    if (nseg <= 1) return;
    const int64_t seglen = ceil_div(ceil_div(s.L, nseg), kStateChunk) * kStateChunk;
    *seglen_out = seglen;
    *nseg_out = (int)ceil_div(s.L, seglen);
}

int scan_fwd_segments(const LaunchShape &s, int paths) {
    int nseg;
    int64_t seglen;
    seg_plan(s, paths, 32, &nseg, &seglen);
    return nseg;
}

size_t scan_fwd_workspace_bytes(const LaunchShape &s, int paths) {
    const int nseg = scan_fwd_segments(s, paths);
    if (nseg <= 1) return 0;
    return (size_t)s.B * paths * s.D * nseg * 2 * s.N * sizeof(float);
}

template <int NS, typename Tin, typename Tout, int MODE, bool VEC>
static cudaError_t launch_ns(const FwdParams &p, cudaStream_t stream) {
    dim3 grid((unsigned)ceil_div(p.D, kWarp), MODE == kModeBidir ? 2 : kPaths, (unsigned)(p.B * p.nseg));
    if (p.nseg == 1) {
        scan_fwd_kernel<NS, Tin, Tout, MODE, 0, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
    } else {
        scan_fwd_kernel<NS, Tin, Tout, MODE, 1, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
        scan_fwd_kernel<NS, Tin, Tout, MODE, 2, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
    }
    return cudaGetLastError();
}

template <typename Tin, typename Tout, int MODE, bool VEC>
static cudaError_t launch_types(const FwdParams &p, cudaStream_t stream) {
    if (p.N <= 4) return launch_ns<4, Tin, Tout, MODE, VEC>(p, stream);
    if (p.N <= 8) return launch_ns<8, Tin, Tout, MODE, VEC>(p, stream);
    return launch_ns<16, Tin, Tout, MODE, VEC>(p, stream);
}

template <int MODE, bool VEC>
static cudaError_t launch_mode(const FwdParams &p, ss2d_dtype_t din, ss2d_dtype_t dout, cudaStream_t stream) {
    if (din == SS2D_F32 && dout == SS2D_F32) return launch_types<float, float, MODE, VEC>(p, stream);
    if (din == SS2D_F32) return launch_types<float, __nv_bfloat16, MODE, VEC>(p, stream);
    if (dout == SS2D_F32) return launch_types<__nv_bfloat16, float, MODE, VEC>(p, stream);
    return launch_types<__nv_bfloat16, __nv_bfloat16, MODE, VEC>(p, stream);
}

cudaError_t launch_scan_fwd(const LaunchShape &s, const ScanFwdArgs &a, void *workspace, cudaStream_t stream) {
    FwdParams p;
    p.u = a.u;
    p.uT = a.uT;
    p.delta = a.delta;
    p.A = a.A;
    p.Bm = a.Bm;
    p.Cm = a.Cm;
    p.Dv = a.Dv;
    p.bias = a.bias;
    p.out = a.out;
    p.chunk_states = a.chunk_states;
    const bool seq = !a.from_image && !a.bidir;
    p.z = seq ? a.z : nullptr;
    p.last_state = seq ? a.last_state : nullptr;
    p.seg = static_cast<float *>(workspace);
    p.xdbl = a.xdbl;
    p.Wdt = a.Wdt;
    p.R = a.R;
    p.B = s.B;
    p.D = s.D;
    p.H = s.H;
    p.W = s.W;
    p.L = s.L;
    p.N = (int)s.N;
    p.softplus = a.softplus;
    seg_plan(s, a.bidir ? 2 : kPaths, a.max_segments, &p.nseg, &p.seglen);
    p.nchunks = ceil_div(s.L, kStateChunk);
    // 4-step vector loads need every row start and step group 4-element aligned
    const bool vec = (s.L % 4) == 0;
    if (a.bidir) {  // the merge that follows reads fp32 per-direction outputs
        if (a.in_dtype == SS2D_F32)
            return vec ? launch_types<float, float, kModeBidir, true>(p, stream)
                       : launch_types<float, float, kModeBidir, false>(p, stream);
        return vec ? launch_types<__nv_bfloat16, float, kModeBidir, true>(p, stream)
                   : launch_types<__nv_bfloat16, float, kModeBidir, false>(p, stream);
    }
    if (a.from_image && a.xdbl) {  // producer fused: fp32 per-path outputs for the merge
        if (!a.delta) {  // dt projected in the scan
            if (a.in_dtype == SS2D_F32)
                return vec ? launch_types<float, float, kModeImgProj, true>(p, stream)
                           : launch_types<float, float, kModeImgProj, false>(p, stream);
            return vec ? launch_types<__nv_bfloat16, float, kModeImgProj, true>(p, stream)
                       : launch_types<__nv_bfloat16, float, kModeImgProj, false>(p, stream);
        }
        if (a.in_dtype == SS2D_F32)
            return vec ? launch_types<float, float, kModeImgProjWide, true>(p, stream)
                       : launch_types<float, float, kModeImgProjWide, false>(p, stream);
        return vec ? launch_types<__nv_bfloat16, float, kModeImgProjWide, true>(p, stream)
                   : launch_types<__nv_bfloat16, float, kModeImgProjWide, false>(p, stream);
    }
    if (a.from_image)
        return vec ? launch_mode<kModeImg, true>(p, a.in_dtype, a.out_dtype, stream)
                   : launch_mode<kModeImg, false>(p, a.in_dtype, a.out_dtype, stream);
    return vec ? launch_mode<kModeSeq, true>(p, a.in_dtype, a.out_dtype, stream)
               : launch_mode<kModeSeq, false>(p, a.in_dtype, a.out_dtype, stream);
}

}  // namespace ss2d
