// Backward pass of one direction of the TTT-MLP scan (fp32 state and
// gradients, tf32 tensor-core products; any b <= 64, d = 16, 32 or 64): given
// dZ = dLoss/dz for every token, the gradients with respect to the token
// streams Q, K, V and the initial state W1_0, W2_0.
//
// The forward chunk (paper notes page, "关键设计 / TTT-MLP 层"; n tokens in
// walking order, state W1 [m x d], W2 [d x m] at the chunk start, rows of the
// matrices below are tokens, tril keeps s <= t in walking order):
//   A = K W1^T, G = GELU(A), Y = G W2^T, D2 = -2 eta (Y - V), P = D2 W2,
//   Dl = P * GELU'(A),  W1' = W1 + Dl^T K,  W2' = W2 + D2^T G,
//   Mk = tril(Q K^T), Aq = Q W1^T + Mk Dl, Gq = GELU(Aq),
//   Ng = tril(Gq G^T), Z = Gq W2^T + Ng D2
// is differentiated by hand (reverse-mode chain rule; GELU'' = phi (2 - a^2)),
// given dZ of the chunk and the gradient with respect to the chunk-end state
// (carried backward from the next chunk):
//   dW2 += dZ^T Gq,  dGq = dZ W2 + tril(dZ D2^T) G,  dD2 = Ng^T dZ,  dG = tril(dZ D2^T)^T Gq,
//   dAq = dGq * GELU'(Aq),  dQ = dAq W1 + tril(dAq Dl^T) K,  dK = tril(dAq Dl^T)^T Q,
//   dDl = Mk^T dAq + K dW1'^T,  dK += Dl dW1',  dD2 += G dW2'^T,  dG += D2 dW2',
//   dP = dDl * GELU'(A),  dA = dDl * P * GELU''(A),  dD2 += dP W2^T,
//   dE = -2 eta dD2,  dV = -dE,  dG += dE W2,  dA += dG * GELU'(A),  dK += dA W1,
//   dW1 = dW1' + dAq^T Q + dA^T K,  dW2 = dW2' + dZ^T Gq + D2^T dP + dE^T G.
// The chunk-start states come from checkpoints: the kernel first walks the
// sequence forward (state updates only) keeping the state every kCkpt chunks,
// then, from the end, runs the chunks' backward steps in reverse, each
// segment's chunk-start states rebuilt from its checkpoint first when kCkpt > 1.
// By default (kCkpt = 1) the walk keeps every chunk-start state ((T / b) 2 m d
// floats per head), writing each state update straight into the next chunk's
// slot, and the backward steps read the states in place.  (Keeping each
// chunk's A, G, P and D2 too, 50 GB more at 313,344 tokens, measured no
// faster: the reads from HBM cost what the recomputation did.)
//
// One cluster of CS CTAs of 512 threads per head (CS = 1 or 2); the matrices of
// a chunk live in a per-head scratch area in global memory (it stays in L2);
// every product is a block GEMM tiled through shared memory whose output tiles
// are dealt out over the cluster's CTAs, and every elementwise pass strides over
// all of the cluster's threads, with a cluster barrier (release / acquire) where
// the CTAs' results meet: after each group of products that do not depend on
// one another, and after each pass.  dE = -2 eta dD2 is never formed: the
// products that read it take -2 eta as their alpha.  Each output element is
// computed by the same sequence of operations whatever CS is, so the results
// do not depend on it.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int NT = 512;          // threads per CTA
constexpr int BMAX = 64;         // largest chunk
// Chunks between two checkpoints.  1: every chunk-start state is kept (128 KB per chunk and head at
// d = 64), so nothing is rebuilt; larger spacings trade that memory for a rebuild of each segment.
#ifndef TTT_BWD_CKPT
#define TTT_BWD_CKPT 1
#endif
constexpr int kCkpt = TTT_BWD_CKPT;

struct BwdArgs {
    const float* Q;
    const float* K;
    const float* V;
    long long qkv_hs, qkv_ts;
    const float* dZ;             // [tokens] in the X layout
    long long x_hs, x_ts;
    const float* W1_0;           // [H, m, d]
    const float* W2_0;           // [H, d, m]
    float* dQ;                   // qkv layout (written)
    float* dK;
    float* dV;
    float* dW1;                  // [H, m, d] (accumulated)
    float* dW2;                  // [H, d, m] (accumulated)
    float* scratch;              // per head: scratch_per_head floats
    long long scratch_per_head;
    int T, H, d, b, reverse;
    float eta;
    int split_tf32;              // products in the split (fp32-accurate) form; else single tf32
};

// Per-head scratch layout (floats).
struct Scratch {
    float *W1, *W2;              // running state
    float *dW1, *dW2;            // carried state gradient
    float *ck;                   // checkpoints: [nck][2 m d]
    float *seg;                  // chunk-start states of one segment: [kCkpt][2 m d]
    // chunk matrices
    float *Qc, *Kc, *Vc, *dZc;                 // [n x d]
    float *A, *G, *P, *Dl, *Aq, *Gq;           // [n x m]
    float *dA, *dG, *dGq, *dDl;                // [n x m]
    float *GpA;                                // GELU'(A) [n x m]
    float *D2, *dD2, *dQc, *dKc;               // [n x d]
    float *Mk, *Ng, *dNg, *dMk;                // [n x n]
};

__host__ __device__ inline long long scratch_floats_for(int d, int b, int T) {
    const long long m = 4LL * d, md = m * d;
    const long long nch = (T + b - 1) / b, nck = (nch + kCkpt - 1) / kCkpt;
    return 4 * md + nck * 2 * md + kCkpt * 2 * md + 4LL * BMAX * d + 11LL * BMAX * m + 4LL * BMAX * d +
           4LL * BMAX * BMAX + 64;
}

__device__ Scratch carve(float* base, int d, int nck) {
    const long long m = 4LL * d, md = m * d;
    Scratch s;
    float* p = base;
    s.W1 = p; p += md;
    s.W2 = p; p += md;
    s.dW1 = p; p += md;
    s.dW2 = p; p += md;
    s.ck = p; p += (long long)nck * 2 * md;
    s.seg = p; p += (long long)kCkpt * 2 * md;
    s.Qc = p; p += BMAX * d;
    s.Kc = p; p += BMAX * d;
    s.Vc = p; p += BMAX * d;
    s.dZc = p; p += BMAX * d;
    s.A = p; p += BMAX * m;
    s.G = p; p += BMAX * m;
    s.P = p; p += BMAX * m;
    s.Dl = p; p += BMAX * m;
    s.Aq = p; p += BMAX * m;
    s.Gq = p; p += BMAX * m;
    s.dA = p; p += BMAX * m;
    s.dG = p; p += BMAX * m;
    s.dGq = p; p += BMAX * m;
    s.dDl = p; p += BMAX * m;
    s.GpA = p; p += BMAX * m;
    s.D2 = p; p += BMAX * d;
    s.dD2 = p; p += BMAX * d;
    s.dQc = p; p += BMAX * d;
    s.dKc = p; p += BMAX * d;
    s.Mk = p; p += BMAX * BMAX;
    s.Ng = p; p += BMAX * BMAX;
    s.dNg = p; p += BMAX * BMAX;
    s.dMk = p; p += BMAX * BMAX;
    return s;
}

// The barrier between the stages of a head: the CTA's own with one CTA per head, else the cluster's
// (release / acquire at cluster scope, so the other CTAs' global-memory results are visible after it).
// Every thread of every CTA of the cluster reaches the same sequence of these.
__device__ __forceinline__ void head_sync(int ncta) {
    if (ncta == 1)
        __syncthreads();
    else
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A matrix operand: element (r, c) of op(X) at X[r * rs + c * cs].
struct Mat {
    const float* p;
    int rs, cs;
};
__device__ __forceinline__ Mat N_(const float* p, int ld) { return Mat{p, ld, 1}; }   // row-major as is
__device__ __forceinline__ Mat T_(const float* p, int ld) { return Mat{p, 1, ld}; }   // transposed view

// C[M x N] (+)= alpha * A[M x Kd] B[Kd x N], C row-major with leading dimension ldc.
// mask: 0 none, 1 keep C[r][c] only for c <= r (lower triangle incl. diagonal).
// All threads of the head's CTAs call it; it ends with the head's barrier.
//
// The products are small (at most 64 x 256 outputs, a reduction of at most 256) and each waits on the
// previous one, so what sets their time is the number of dependent memory round trips, not arithmetic:
// the operands' reduction blocks (KB deep) are copied into shared memory by cp.async (16-byte copies
// that bypass L1 and zero-fill past the matrices' edges), NSTAGE blocks in flight at once, and an
// accumulating product loads its old C before the reduction starts, so a product with a reduction of
// at most 96 costs one round trip for its inputs and one for its stores.
//
// Arithmetic: mma.sync m16n8k8 on tf32 operands in the split form ("3xTF32"): each operand
// x = hi + lo with hi = tf32(x) and lo = tf32(x - hi), and a b is taken as a_hi b_hi + a_hi b_lo +
// a_lo b_hi, the small terms first; the dropped a_lo b_lo and the rounding of lo leave about 2^-21 of
// |a b|, fp32 accuracy for these sums.  16 warps in a grid of WM x WN warp tiles.  Staging: an operand
// whose reduction index is contiguous in memory is kept as [row][KB + 4] in shared memory, otherwise as
// [k][rows + 8]; either way the fragment loads (lanes g = lane / 4 along rows, t = lane % 4 along k)
// fall in 32 distinct banks and the 16-byte copies run along the contiguous index.
constexpr int KB = 32;
constexpr int NSTAGE = 4;
constexpr int PADK = 4, PADR = 8;
__host__ __device__ constexpr int stage_floats(int rows) {
    return rows * (KB + PADK) > KB * (rows + PADR) ? rows * (KB + PADK) : KB * (rows + PADR);
}
// dynamic shared memory of the kernel: the largest tile pair of the head's CTA count, NSTAGE times
__host__ __device__ constexpr int gemm_smem_floats(int ncta) {
    return NSTAGE * (ncta == 1 ? stage_floats(64) + stage_floats(256) : stage_floats(64) + stage_floats(128));
}

__device__ __forceinline__ void cp_async16(float* dst, const float* src, int bytes) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ int clamp4(int x) { return x < 0 ? 0 : (x > 4 ? 4 : x); }

__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float r = x - __uint_as_float(hi);   // exact: x and hi agree in their leading bits
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

// SPLIT: hi and lo as above; else hi = tf32(x) alone (lo unused)
template <bool SPLIT>
__device__ __forceinline__ void to_tf32(float x, uint32_t& hi, uint32_t& lo) {
    if constexpr (SPLIT) {
        split_tf32(x, hi, lo);
    } else {
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
        lo = 0;
    }
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Copies reduction block [k0, k0 + KB) of a ROWS-row operand X (element (r, k) of the operand at
// X.at(r, k) when X is A; at X.at(k, r) when X is B, i.e. B's columns are its rows here) into stage
// buffer st.  KMAJ: the reduction index is contiguous in memory.
template <int ROWS, bool KMAJ>
__device__ __forceinline__ void stage_operand(float* st, const float* p, long long rstride, long long kstride,
                                              int r0, int R, int k0, int Kd, int tid) {
    if constexpr (KMAJ) {   // 16 bytes = 4 consecutive k of one row; layout [row][KB + PADK]
        for (int e = tid; e < ROWS * (KB / 4); e += NT) {
            const int rr = e / (KB / 4), kq = (e % (KB / 4)) * 4;
            const int gr = r0 + rr, gk = k0 + kq;
            const int bytes = gr < R ? 4 * clamp4(Kd - gk) : 0;
            cp_async16(st + rr * (KB + PADK) + kq, bytes ? p + gr * rstride + gk : p, bytes);
        }
    } else {      // 16 bytes = 4 consecutive rows at one k; layout [k][ROWS + PADR]
        for (int e = tid; e < KB * (ROWS / 4); e += NT) {
            const int kk = e / (ROWS / 4), rq = (e % (ROWS / 4)) * 4;
            const int gr = r0 + rq, gk = k0 + kk;
            const int bytes = gk < Kd ? 4 * clamp4(R - gr) : 0;
            cp_async16(st + kk * (ROWS + PADR) + rq, bytes ? p + gr + gk * kstride : p, bytes);
        }
    }
}

// A_K / B_K: the operand's reduction index is contiguous in memory (A.cs == 1 / B.rs == 1), which fixes
// its staging layout at compile time, so that every fragment load is one shared load at a constant
// offset from a per-thread base.
template <int BM, int BN, int WM, int WN, bool SPLIT, bool A_K, bool B_K>
__device__ __noinline__ void gemm_tiles(float* C, int ldc, const Mat& A, const Mat& B, int M, int N, int Kd,
                                        float alpha, bool accumulate, const float* Cin, int mask, bool bar, int rank,
                                        int ncta, float* smem) {
    constexpr int WGN = BN / WN;
    static_assert((BM / WM) * WGN == NT / 32, "warp grid");
    static_assert(WM % 16 == 0 && WN % 8 == 0 && BM % 4 == 0 && BN % 4 == 0, "warp tile");
    constexpr int MT = WM / 16, NTL = WN / 8;
    constexpr int SA = stage_floats(BM), STAGE = SA + stage_floats(BN);
    static_assert(STAGE * NSTAGE <= gemm_smem_floats(BM + BN > 192 ? 1 : 2), "staging");
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int g = lane / 4, t = lane % 4;
    const int wr = (warp / WGN) * WM, wc = (warp % WGN) * WN;
    // A (r, k) = A.p[r rs + k cs]; B's column n at k: B.p[k rs + n cs]
    const long long a_rstr = A_K ? A.rs : 1, a_kstr = A_K ? 1 : A.cs;
    const long long b_rstr = B_K ? B.cs : 1, b_kstr = B_K ? 1 : B.rs;
    // staged element (row, k) of A at a_base + row * A_RS + k * A_KS (B likewise), relative to this
    // thread's first fragment element (row wr + g or wc + g, k = t)
    constexpr int A_RS = A_K ? KB + PADK : 1, A_KS = A_K ? 1 : BM + PADR;
    constexpr int B_RS = B_K ? KB + PADK : 1, B_KS = B_K ? 1 : BN + PADR;
    const int a_base = (wr + g) * A_RS + t * A_KS;
    const int b_base = SA + (wc + g) * B_RS + t * B_KS;
    const int nkb = (Kd + KB - 1) / KB;
    int tile = 0;
    bool first = true;   // the call starts behind the head's barrier: the staging is free
    for (int m0 = 0; m0 < M; m0 += BM) {
        for (int n0 = 0; n0 < N; n0 += BN) {
            if (tile++ % ncta != rank) continue;   // another CTA of the cluster owns this tile
            if (!first) __syncthreads();           // the previous tile's reads of the staging are done
            first = false;
            auto row_of = [&](int i, int q) { return m0 + wr + i * 16 + g + (q >= 2 ? 8 : 0); };
            auto col_of = [&](int j, int q) { return n0 + wc + j * 8 + 2 * t + (q & 1); };
            auto issue = [&](int kb) {
                float* st = smem + (kb % NSTAGE) * STAGE;
                stage_operand<BM, A_K>(st, A.p, a_rstr, a_kstr, m0, M, kb * KB, Kd, tid);
                stage_operand<BN, B_K>(st + SA, B.p, b_rstr, b_kstr, n0, N, kb * KB, Kd, tid);
            };
#pragma unroll
            for (int sidx = 0; sidx < NSTAGE - 1; ++sidx) {
                if (sidx < nkb) issue(sidx);
                cp_async_commit();
            }
            // accumulators q and q + 1 (q even) are neighbours in a row of C: one 8-byte access (ldc and the
            // column are even) unless the pair straddles the last column
            float acc[MT][NTL][4], cold[MT][NTL][4];
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int j = 0; j < NTL; ++j)
#pragma unroll
                    for (int q = 0; q < 4; q += 2) {
                        acc[i][j][q] = acc[i][j][q + 1] = 0.f;
                        cold[i][j][q] = cold[i][j][q + 1] = 0.f;
                        const int r = row_of(i, q), c = col_of(j, q);
                        if (!accumulate || r >= M || c >= N) continue;
                        const float* src = Cin + (long long)r * ldc + c;
                        if (c + 1 < N) {
                            const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
                            cold[i][j][q] = v.x;
                            cold[i][j][q + 1] = v.y;
                        } else {
                            cold[i][j][q] = __ldcg(src);
                        }
                    }
            for (int kb = 0; kb < nkb; ++kb) {
                cp_async_wait<NSTAGE - 2>();   // block kb has landed (this thread's copies)
                __syncthreads();               // everyone's copies, and block kb - 1's products are done
                if (kb + NSTAGE - 1 < nkb) issue(kb + NSTAGE - 1);
                cp_async_commit();
                const float* sta = smem + (kb % NSTAGE) * STAGE + a_base;
                const float* stb = smem + (kb % NSTAGE) * STAGE + b_base;
#pragma unroll
                for (int k8 = 0; k8 < KB; k8 += 8) {
                    uint32_t ah[MT][4], al[MT][4];
#pragma unroll
                    for (int i = 0; i < MT; ++i) {
                        const float* pa = sta + i * 16 * A_RS + k8 * A_KS;
                        to_tf32<SPLIT>(pa[0], ah[i][0], al[i][0]);
                        to_tf32<SPLIT>(pa[8 * A_RS], ah[i][1], al[i][1]);
                        to_tf32<SPLIT>(pa[4 * A_KS], ah[i][2], al[i][2]);
                        to_tf32<SPLIT>(pa[8 * A_RS + 4 * A_KS], ah[i][3], al[i][3]);
                    }
#pragma unroll
                    for (int j = 0; j < NTL; ++j) {
                        const float* pb = stb + j * 8 * B_RS + k8 * B_KS;
                        uint32_t bh0, bl0, bh1, bl1;
                        to_tf32<SPLIT>(pb[0], bh0, bl0);
                        to_tf32<SPLIT>(pb[4 * B_KS], bh1, bl1);
#pragma unroll
                        for (int i = 0; i < MT; ++i) {
                            if constexpr (SPLIT) {
                                mma_tf32(acc[i][j], al[i], bh0, bh1);
                                mma_tf32(acc[i][j], ah[i], bl0, bl1);
                            }
                            mma_tf32(acc[i][j], ah[i], bh0, bh1);
                        }
                    }
                }
            }
            cp_async_wait<0>();
            // accumulator q of warp tile (i, j): row wr + 16 i + g (+ 8 for q >= 2), column wc + 8 j + 2 t (+ 1 if q odd)
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int j = 0; j < NTL; ++j)
#pragma unroll
                    for (int q = 0; q < 4; q += 2) {
                        const int r = row_of(i, q), c = col_of(j, q);
                        if (r >= M || c >= N) continue;
                        const float v0 = (mask == 1 && c > r ? 0.f : alpha * acc[i][j][q]) + cold[i][j][q];
                        const float v1 = (mask == 1 && c + 1 > r ? 0.f : alpha * acc[i][j][q + 1]) + cold[i][j][q + 1];
                        float* dst = C + (long long)r * ldc + c;
                        if (c + 1 < N)
                            *reinterpret_cast<float2*>(dst) = make_float2(v0, v1);
                        else
                            *dst = v0;
                    }
        }
    }
    if (bar)
        head_sync(ncta);
    else
        __syncthreads();   // only the staging is reused by the CTA's next product
}

// Tile shapes: one CTA tile covers a whole b x m (or m x d) product when the head has one CTA, half of
// it per CTA with two; the b x b and b x d products take 64 x 64 tiles (32 x 64 with two CTAs).
template <int BM, int BN, int WM, int WN, bool SPLIT>
__device__ __forceinline__ void gemm_major(float* C, int ldc, const Mat& A, const Mat& B, int M, int N, int Kd,
                                           float alpha, bool accumulate, const float* Cin, int mask, bool bar,
                                           int rank, int ncta, float* sm) {
    if (A.cs == 1) {
        if (B.rs == 1)
            gemm_tiles<BM, BN, WM, WN, SPLIT, true, true>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
        else
            gemm_tiles<BM, BN, WM, WN, SPLIT, true, false>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
    } else {
        if (B.rs == 1)
            gemm_tiles<BM, BN, WM, WN, SPLIT, false, true>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
        else
            gemm_tiles<BM, BN, WM, WN, SPLIT, false, false>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar,
                                                              rank, ncta, sm);
    }
}

template <bool SPLIT>
__device__ __forceinline__ void gemm_shapes(float* C, int ldc, const Mat& A, const Mat& B, int M, int N, int Kd,
                                            float alpha, bool accumulate, const float* Cin, int mask, bool bar,
                                            int rank, int ncta, float* sm) {
    if (ncta == 1) {
        if (N > 64 && M <= 64)
            gemm_major<64, 256, 16, 64, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, 0, 1, sm);
        else if (M > 64 && N <= 64)
            gemm_major<256, 64, 32, 32, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, 0, 1, sm);
        else
            gemm_major<64, 64, 16, 16, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, 0, 1, sm);
    } else {
        if (N > 64 && M <= 64)
            gemm_major<64, 128, 16, 32, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
        else if (M > 64 && N <= 64)
            gemm_major<128, 64, 16, 32, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
        else
            gemm_major<32, 64, 16, 8, SPLIT>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin, mask, bar, rank, ncta, sm);
    }
}

// split: the split ("3xTF32", fp32-accurate) products; else single tf32 products (one MMA instead of three)
// Cin: where an accumulating product reads its old C (null: C itself).  bar: end with the head's barrier;
// false only where the next products of the head read nothing this one writes and write nothing it reads
// (a later accumulation into the same C by a product of the same shape is fine: the same threads own the
// same elements of C).
__device__ __noinline__ void gemm_cs(float* C, int ldc, Mat A, Mat B, int M, int N, int Kd, float alpha,
                                     bool accumulate, const float* Cin, int mask, bool bar, int rank, int ncta,
                                     bool split) {
    extern __shared__ __align__(16) float dyn_smem[];
    if (split)
        gemm_shapes<true>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin ? Cin : C, mask, bar, rank, ncta, dyn_smem);
    else
        gemm_shapes<false>(C, ldc, A, B, M, N, Kd, alpha, accumulate, Cin ? Cin : C, mask, bar, rank, ncta, dyn_smem);
}

__device__ __forceinline__ float gelu_pp(float a) {   // GELU''(a) = phi(a) (2 - a^2)
    return 0.39894228040143268f * expf(-0.5f * a * a) * (2.0f - a * a);
}

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles between stage boundaries seen by thread 0 of CTA 0 (16 slots).
__device__ long long* g_dbg_bwd = nullptr;
#define STAMPB(k)                                           \
    do {                                                    \
        if (tid == 0 && blockIdx.x == 0) {                  \
            const long long now_ = clock64();               \
            stamp_acc[k] += now_ - stamp_last;              \
            stamp_last = now_;                              \
        }                                                   \
    } while (0)
#else
#define STAMPB(k) \
    do {          \
    } while (0)
#endif

template <int D, int CS>
__global__ void __launch_bounds__(NT, 1) scan_bwd_kernel(BwdArgs a) {
    constexpr int M = 4 * D;
    constexpr long long MD = (long long)M * D;
    constexpr int GNT = CS * NT;   // threads of the head's cluster
    int rank = 0;
    if constexpr (CS > 1) asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int h = blockIdx.x / CS, tid = threadIdx.x, gtid = rank * NT + tid;
    // a product of the head, its output tiles dealt out over the cluster (ends with the head's barrier)
    auto gemm = [&](float* C, int ldc, Mat A_, Mat B_, int M_, int N_, int Kd, float alpha, bool accumulate,
                    int mask = 0, const float* Cin = nullptr) {
        gemm_cs(C, ldc, A_, B_, M_, N_, Kd, alpha, accumulate, Cin, mask, true, rank, CS, a.split_tf32 != 0);
    };
    // the same, without the head's barrier: for a product whose successors up to the next barrier are
    // independent of it
    auto gemm_nb = [&](float* C, int ldc, Mat A_, Mat B_, int M_, int N_, int Kd, float alpha, bool accumulate,
                       int mask = 0, const float* Cin = nullptr) {
        gemm_cs(C, ldc, A_, B_, M_, N_, Kd, alpha, accumulate, Cin, mask, false, rank, CS, a.split_tf32 != 0);
    };
    auto sync = [&]() { head_sync(CS); };
    const int T = a.T, b = a.b;
    const int nch = (T + b - 1) / b, nck = (nch + kCkpt - 1) / kCkpt;
    Scratch s = carve(a.scratch + (long long)h * a.scratch_per_head, D, nck);
    const float eta = a.eta;

#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[16] = {};
    long long stamp_last = clock64();
#endif
    auto token = [&](int c, int r) { return a.reverse ? T - 1 - (c * b + r) : c * b + r; };
    auto load_chunk = [&](int c, int n, bool with_q, bool with_dz) {
        const float* __restrict__ gK = a.K;
        const float* __restrict__ gV = a.V;
        const float* __restrict__ gQ = a.Q;
        const float* __restrict__ gdZ = a.dZ;
        float* __restrict__ Kc = s.Kc;
        float* __restrict__ Vc = s.Vc;
        float* __restrict__ Qc = s.Qc;
        float* __restrict__ dZc = s.dZc;
#pragma unroll 4
        for (int idx = gtid; idx < n * D; idx += GNT) {
            const int r = idx / D, j = idx % D;
            const long long off = (long long)h * a.qkv_hs + (long long)token(c, r) * a.qkv_ts + j;
            Kc[idx] = gK[off];
            Vc[idx] = gV[off];
            if (with_q) Qc[idx] = gQ[off];
            if (with_dz) dZc[idx] = gdZ[(long long)h * a.x_hs + (long long)token(c, r) * a.x_ts + j];
        }
        sync();
    };
    // A = K W1^T, G = GELU(A), D2 = -2 eta (G W2^T - V), P = D2 W2, Dl = P GELU'(A)
    // bwd: the backward step's first products that need only the loaded chunk and the state (Mk, Q W1^T,
    // dZ W2) go beside A, and tril(dZ D2^T) beside P
    auto chunk_core = [&](int n, bool bwd) {
        if (bwd) {
            gemm_nb(s.A, M, N_(s.Kc, D), T_(s.W1, D), n, M, D, 1.f, false);
            gemm_nb(s.Mk, BMAX, N_(s.Qc, D), T_(s.Kc, D), n, n, D, 1.f, false, 1);
            gemm_nb(s.Aq, M, N_(s.Qc, D), T_(s.W1, D), n, M, D, 1.f, false);
            gemm(s.dGq, M, N_(s.dZc, D), N_(s.W2, M), n, M, D, 1.f, false);                 // dZ W2
        } else {
            gemm(s.A, M, N_(s.Kc, D), T_(s.W1, D), n, M, D, 1.f, false);
        }
        {   // (restrict views scoped to each loop: several iterations' loads may be in flight)
            const float* __restrict__ A_ = s.A;
            float* __restrict__ G_ = s.G;
#pragma unroll 4
            for (int idx = gtid; idx < n * M; idx += GNT) G_[idx] = gelu(A_[idx]);
        }
        sync();
        gemm(s.D2, D, N_(s.G, M), T_(s.W2, M), n, D, M, 1.f, false);
        {
            float* __restrict__ D2_ = s.D2;
            const float* __restrict__ V_ = s.Vc;
#pragma unroll 4
            for (int idx = gtid; idx < n * D; idx += GNT) D2_[idx] = -2.0f * eta * (D2_[idx] - V_[idx]);
        }
        sync();
        if (bwd) {
            gemm_nb(s.P, M, N_(s.D2, D), N_(s.W2, M), n, M, D, 1.f, false);
            gemm(s.dNg, BMAX, N_(s.dZc, D), T_(s.D2, D), n, n, D, 1.f, false, 1);            // tril(dZ D2^T)
        } else {
            gemm(s.P, M, N_(s.D2, D), N_(s.W2, M), n, M, D, 1.f, false);
        }
        {
            const float* __restrict__ A_ = s.A;
            const float* __restrict__ P_ = s.P;
            float* __restrict__ Dl_ = s.Dl;
            float* __restrict__ Gp_ = s.GpA;
#pragma unroll 4
            for (int idx = gtid; idx < n * M; idx += GNT) {
                float g, gp;
                gelu_and_prime(A_[idx], g, gp);
                Dl_[idx] = P_[idx] * gp;
                if (bwd) Gp_[idx] = gp;   // for the backward step's passes
            }
        }
        sync();
    };
    // W1 += Dl^T K, W2 += D2^T G
    auto chunk_update = [&](int n) {
        gemm(s.W1, D, T_(s.Dl, M), N_(s.Kc, D), M, D, n, 1.f, true);
        gemm(s.W2, M, T_(s.D2, D), N_(s.G, M), D, M, n, 1.f, true);
    };
    // cnt a multiple of 4, both 16-byte aligned: four 16-byte loads in flight per thread before their stores
    auto copy = [&](float* dst, const float* src, long long cnt) {
        const float4* __restrict__ s4 = reinterpret_cast<const float4*>(src);
        float4* __restrict__ d4 = reinterpret_cast<float4*>(dst);
        const long long n4 = cnt / 4;
        for (long long i = gtid; i < n4; i += 4 * GNT) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i + u * GNT < n4) v[u] = s4[i + u * GNT];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i + u * GNT < n4) d4[i + u * GNT] = v[u];
        }
        sync();
    };

    // kCkpt = 1: chunk c's state, in place
    auto point_at_chunk = [&](int c) {
        s.W1 = s.ck + (long long)c * 2 * MD;
        s.W2 = s.W1 + MD;
    };

    // ---- forward walk: checkpoints of the state every kCkpt chunks
    if constexpr (kCkpt == 1) {
        copy(s.ck, a.W1_0 + (long long)h * MD, MD);
        copy(s.ck + MD, a.W2_0 + (long long)h * MD, MD);
    } else {
        copy(s.W1, a.W1_0 + (long long)h * MD, MD);
        copy(s.W2, a.W2_0 + (long long)h * MD, MD);
    }
    for (int c = 0; c < nch; ++c) {
        const int n = min(b, T - c * b);
        if constexpr (kCkpt == 1) {
            point_at_chunk(c);
        } else if (c % kCkpt == 0) {
            copy(s.ck + (long long)(c / kCkpt) * 2 * MD, s.W1, MD);
            copy(s.ck + (long long)(c / kCkpt) * 2 * MD + MD, s.W2, MD);
        }
        STAMPB(0);
        load_chunk(c, n, false, false);
        STAMPB(1);
        chunk_core(n, false);
        STAMPB(2);
        if constexpr (kCkpt == 1) {   // the next chunk's state = this one's + the update (the last is not needed)
            if (c + 1 < nch) {
                float* W1n = s.ck + (long long)(c + 1) * 2 * MD;
                gemm_nb(W1n, D, T_(s.Dl, M), N_(s.Kc, D), M, D, n, 1.f, true, 0, s.W1);
                gemm(W1n + MD, M, T_(s.D2, D), N_(s.G, M), D, M, n, 1.f, true, 0, s.W2);
            }
        } else {
            chunk_update(n);
        }
        STAMPB(3);
    }

    // ---- backward, segment by segment from the end
    for (long long i = gtid; i < MD; i += GNT) { s.dW1[i] = 0.f; s.dW2[i] = 0.f; }
    sync();
    for (int sg = nck - 1; sg >= 0; --sg) {
        const int c0 = sg * kCkpt, c1 = min(nch, c0 + kCkpt);
        if constexpr (kCkpt > 1) {
        copy(s.W1, s.ck + (long long)sg * 2 * MD, MD);
        copy(s.W2, s.ck + (long long)sg * 2 * MD + MD, MD);
        STAMPB(4);
        for (int c = c0; c < c1; ++c) {   // chunk-start states of the segment
            copy(s.seg + (long long)(c - c0) * 2 * MD, s.W1, MD);
            copy(s.seg + (long long)(c - c0) * 2 * MD + MD, s.W2, MD);
            STAMPB(4);
            if (c + 1 < c1) {
                const int n = min(b, T - c * b);
                load_chunk(c, n, false, false);
                chunk_core(n, false);
                chunk_update(n);
            }
            STAMPB(5);
        }
        }
        for (int c = c1 - 1; c >= c0; --c) {
            const int n = min(b, T - c * b);
            if constexpr (kCkpt > 1) {
                copy(s.W1, s.seg + (long long)(c - c0) * 2 * MD, MD);
                copy(s.W2, s.seg + (long long)(c - c0) * 2 * MD + MD, MD);
            } else {   // the chunk's state, kept by the walk: read in place
                point_at_chunk(c);
            }
            STAMPB(6);
            load_chunk(c, n, true, true);
            STAMPB(7);
            // forward intermediates (and the first products of the output branch)
            chunk_core(n, true);
            STAMPB(8);
            gemm_nb(s.Aq, M, N_(s.Mk, BMAX), N_(s.Dl, M), n, M, n, 1.f, true);              // Aq += Mk Dl
            gemm(s.dGq, M, N_(s.dNg, BMAX), N_(s.G, M), n, M, n, 1.f, true);                 // + dNg G
            {   // Gq = GELU(Aq), dAq = dGq GELU'(Aq) (in dGq)
                const float* __restrict__ Aq_ = s.Aq;
                float* __restrict__ Gq_ = s.Gq;
                float* __restrict__ dGq_ = s.dGq;
#pragma unroll 4
                for (int idx = gtid; idx < n * M; idx += GNT) {
                    const float aq = Aq_[idx];
                    float g, gp;
                    gelu_and_prime(aq, g, gp);
                    Gq_[idx] = gelu(aq);
                    dGq_[idx] *= gp;
                }
            }
            sync();
            STAMPB(9);
            // output branch
            gemm_nb(s.Ng, BMAX, N_(s.Gq, M), T_(s.G, M), n, n, M, 1.f, false, 1);            // tril(Gq G^T)
            gemm_nb(s.dG, M, T_(s.dNg, BMAX), N_(s.Gq, M), n, M, n, 1.f, false);             // dNg^T Gq
            gemm_nb(s.dQc, D, N_(s.dGq, M), N_(s.W1, D), n, D, M, 1.f, false);               // dAq W1
            gemm_nb(s.dMk, BMAX, N_(s.dGq, M), T_(s.Dl, M), n, n, M, 1.f, false, 1);         // tril(dAq Dl^T)
            gemm(s.dDl, M, T_(s.Mk, BMAX), N_(s.dGq, M), n, M, n, 1.f, false);               // Mk^T dAq
            STAMPB(10);
            gemm_nb(s.dD2, D, T_(s.Ng, BMAX), N_(s.dZc, D), n, D, n, 1.f, false);            // Ng^T dZ
            gemm_nb(s.dQc, D, N_(s.dMk, BMAX), N_(s.Kc, D), n, D, n, 1.f, true);             // + dMk K
            gemm_nb(s.dKc, D, T_(s.dMk, BMAX), N_(s.Qc, D), n, D, n, 1.f, false);            // dMk^T Q
            // the chunk-end state gradient
            gemm_nb(s.dDl, M, N_(s.Kc, D), T_(s.dW1, D), n, M, D, 1.f, true);               // + K dW1'^T
            gemm_nb(s.dKc, D, N_(s.Dl, M), N_(s.dW1, D), n, D, M, 1.f, true);               // + Dl dW1'
            gemm_nb(s.dD2, D, N_(s.G, M), T_(s.dW2, M), n, D, M, 1.f, true);                // + G dW2'^T
            gemm(s.dG, M, N_(s.D2, D), N_(s.dW2, M), n, M, D, 1.f, true);                   // + D2 dW2'
            // dP (in dDl), dA
            {
                const float* __restrict__ A_ = s.A;
                const float* __restrict__ P_ = s.P;
                const float* __restrict__ Gp_ = s.GpA;
                float* __restrict__ dDl_ = s.dDl;
                float* __restrict__ dA_ = s.dA;
#pragma unroll 4
                for (int idx = gtid; idx < n * M; idx += GNT) {
                    const float ddl = dDl_[idx];
                    dA_[idx] = ddl * P_[idx] * gelu_pp(A_[idx]);
                    dDl_[idx] = ddl * Gp_[idx];
                }
            }
            sync();
            // dE = -2 eta dD2 is applied as the products' alpha (dD2 itself is kept)
            gemm(s.dD2, D, N_(s.dDl, M), T_(s.W2, M), n, D, M, 1.f, true);                  // + dP W2^T
            gemm(s.dG, M, N_(s.dD2, D), N_(s.W2, M), n, M, D, -2.0f * eta, true);           // + dE W2
            {                                                                                // dA += dG GELU'(A)
                const float* __restrict__ Gp_ = s.GpA;
                const float* __restrict__ dG_ = s.dG;
                float* __restrict__ dA_ = s.dA;
#pragma unroll 4
                for (int idx = gtid; idx < n * M; idx += GNT) dA_[idx] += dG_[idx] * Gp_[idx];
            }
            sync();
            STAMPB(11);
            gemm_nb(s.dKc, D, N_(s.dA, M), N_(s.W1, D), n, D, M, 1.f, true);                // + dA W1
            // the chunk-start state gradient (accumulated onto the chunk-end one)
            gemm_nb(s.dW2, M, T_(s.dZc, D), N_(s.Gq, M), D, M, n, 1.f, true);               // dZ^T Gq
            gemm_nb(s.dW2, M, T_(s.D2, D), N_(s.dDl, M), D, M, n, 1.f, true);               // D2^T dP
            gemm_nb(s.dW2, M, T_(s.dD2, D), N_(s.G, M), D, M, n, -2.0f * eta, true);        // dE^T G
            gemm_nb(s.dW1, D, T_(s.dGq, M), N_(s.Qc, D), M, D, n, 1.f, true);               // dAq^T Q
            gemm(s.dW1, D, T_(s.dA, M), N_(s.Kc, D), M, D, n, 1.f, true);                   // dA^T K
            STAMPB(12);
            // dQ, dK, dV of the chunk's tokens
            {
                const float* __restrict__ dQc_ = s.dQc;
                const float* __restrict__ dKc_ = s.dKc;
                const float* __restrict__ dD2_ = s.dD2;
                float* __restrict__ gdQ = a.dQ;
                float* __restrict__ gdK = a.dK;
                float* __restrict__ gdV = a.dV;
#pragma unroll 4
                for (int idx = gtid; idx < n * D; idx += GNT) {
                    const int r = idx / D, j = idx % D;
                    const long long off = (long long)h * a.qkv_hs + (long long)token(c, r) * a.qkv_ts + j;
                    gdQ[off] = dQc_[idx];
                    gdK[off] = dKc_[idx];
                    gdV[off] = dD2_[idx] * (2.0f * eta);   // dV = -dE = 2 eta dD2
                }
            }
            sync();
            STAMPB(13);
        }
    }
#ifdef TTT_DEBUG_STAGES
    if (tid == 0 && blockIdx.x == 0 && g_dbg_bwd) {
        for (int k = 0; k < 16; ++k) g_dbg_bwd[k] = stamp_acc[k];
        g_dbg_bwd[15] = nch;
    }
#endif
    for (long long i = gtid; i < MD; i += GNT) {
        a.dW1[(long long)h * MD + i] += s.dW1[i];
        a.dW2[(long long)h * MD + i] += s.dW2[i];
    }
}

}  // namespace

#ifdef TTT_DEBUG_STAGES
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump_bwd(long long* p) {
    return (int)cudaMemcpyToSymbol(g_dbg_bwd, &p, sizeof(p));
}
#endif

long long scan_backward_scratch_floats(int d, int b, int T) { return scratch_floats_for(d, b, T); }

// CTAs per head of the backward scan: 0 picks (2 while 2 H CTAs fit on the GPU's SMs, else 1); 1 or 2 forces.
static std::atomic<int> g_bwd_cluster{0};

void set_scan_backward_ctas(int ctas) { g_bwd_cluster.store(ctas); }

cudaError_t launch_scan_backward(const float* Q, const float* K, const float* V, long long qkv_hs, long long qkv_ts,
                                 const float* dZ, long long x_hs, long long x_ts, const float* W1_0,
                                 const float* W2_0, float* dQ, float* dK, float* dV, float* dW1, float* dW2,
                                 float* scratch, int T, int H, int d, int b, int reverse, float eta,
                                 int split_tf32, cudaStream_t s) {
    if (b < 1 || b > BMAX) return cudaErrorInvalidValue;
    BwdArgs a{};
    a.Q = Q; a.K = K; a.V = V; a.qkv_hs = qkv_hs; a.qkv_ts = qkv_ts;
    a.dZ = dZ; a.x_hs = x_hs; a.x_ts = x_ts;
    a.W1_0 = W1_0; a.W2_0 = W2_0;
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.dW1 = dW1; a.dW2 = dW2;
    a.scratch = scratch; a.scratch_per_head = scratch_floats_for(d, b, T);
    a.T = T; a.H = H; a.d = d; a.b = b; a.reverse = reverse; a.eta = eta; a.split_tf32 = split_tf32;
    // two CTAs per head while the heads' pairs fit on the GPU at once, else one
    int cs = g_bwd_cluster.load();
    if (cs == 0) {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        cs = 2 * H <= sms ? 2 : 1;
    }
    if (cs != 1 && cs != 2) return cudaErrorInvalidValue;
    void (*kern)(BwdArgs) = nullptr;
    switch (d * 4 + cs) {
        case 16 * 4 + 1: kern = scan_bwd_kernel<16, 1>; break;
        case 32 * 4 + 1: kern = scan_bwd_kernel<32, 1>; break;
        case 64 * 4 + 1: kern = scan_bwd_kernel<64, 1>; break;
        case 16 * 4 + 2: kern = scan_bwd_kernel<16, 2>; break;
        case 32 * 4 + 2: kern = scan_bwd_kernel<32, 2>; break;
        case 64 * 4 + 2: kern = scan_bwd_kernel<64, 2>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(H * cs);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = (size_t)gemm_smem_floats(cs) * sizeof(float);
    cfg.stream = s;
    {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)cfg.dynamicSmemBytes);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope("scan_backward", s);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ttt
