// backward.cu -- the backward pass of the routed MoE block for a given routing.
//
// "Qwen3-VL and Mixture of Experts" (gopikrishnatummala.com), "How the router and experts
// learn", "What gets trained": a token's gradient reaches only the experts it chose, and the
// router learns through the gate weights; the selection is held fixed (piecewise constant).
// For the loss sum_t dy[t] . y[t] and token t with slots j (expert e, weight w_j):
//   z    = W_down[e]^T dy[t]                   dw_j = h . z           dh = w_j z
//   dg   = dh u s (1 + g (1 - s)),  du = dh g s       (s = sigmoid(g), h = g s u)
//   dx  += W_gate[e]^T dg + W_up[e]^T du,     dW_down[e] += (w_j dy) h^T,
//   dW_gate[e] += dg x^T,  dW_up[e] += du x^T,
//   dp_j = (dw_j - sum_m dw_m w_m) / S (renormalised) or dw_j,
//   dl   = p (dp - sum_j p_j dp_j) (+ an added logit gradient, e.g. the balance loss's),
//   dW_r += dl x^T,  db += dl,  dx += W_r^T dl  (+ dy for a residual block).
// z gives both dw and dh, so the down projection is not recomputed; g and u are (one
// grouped GEMM, the same contraction as the forward gate_up).
//
// Work: the forward's router and a stable permutation (tile_m = 1) of the given routing,
// permuted copies of x and dy, then seven grouped bf16 GEMMs with FP32 accumulation on warp
// MMAs (m16n8k16, operands staged in shared memory by cp.async, ldmatrix with or without
// transpose for each operand's major-ness) and small FP32 kernels: the tile and slice tables,
// routing weights per row, the SwiGLU backward, the routing backward, the bias gradient, the
// router-weight gradient's slice sum and the dx sum.  Every sum runs in a fixed order that
// depends only on the shapes: results are bitwise reproducible.  GEMM operands that the
// backward computes (h, dg/du, w dy, dl) are rounded to bf16 once; all outputs are FP32.
#include <algorithm>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

// CTA tile: 128 rows (M) x BN columns (N), K steps of BK, NS-stage cp.async ring; 8 warps as
// 2 (M) x 4 (N), each a 64 x BN/4 warp tile.  Shared-memory rows are padded by 8 elements so
// that the 8 row addresses of every ldmatrix fall in distinct banks.
constexpr int kBwBM = 128, kBwThreads = 256;
constexpr int kBwBN = 128, kBwBK = 64, kBwStages = 3;   // the configuration the library launches
template <int BN, int BK>
struct BwTile {
    static constexpr int RowK = BK + 8;           // [rows][k] tiles
    static constexpr int RowM = kBwBM + 8;        // [k][m] tiles
    static constexpr int RowN = BN + 8;           // [k][n] tiles
    static constexpr int A = kBwBM * RowK > BK * RowM ? kBwBM * RowK : BK * RowM;   // elements
    static constexpr int B = BN * RowK > BK * RowN ? BN * RowK : BK * RowN;
};
template <int BN, int BK, int NS>
constexpr int bw_smem_bytes() { return NS * (BwTile<BN, BK>::A + BwTile<BN, BK>::B) * 2; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    // src-size 0 writes 16 zero bytes and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// One grouped GEMM  C_g[M_g, N] = A_g[M_g, K_g] B_g[K_g, N]  (bf16 in, FP32 out).
// A is stored [m][k] (A_K) or [k][m]; B is stored [n][k] (B_K) or [k][n]; leading dimensions
// in elements, every one a multiple of 8.
// KG = false (grouped along M, the token rows): group g owns rows seg_off[g] ..
//   + seg_cnt[g] of A and C; B advances by b_gs per group; tile_start[g] is g's first
//   128-row tile (groups + 1 entries; NULL: one group of M rows).  K is fixed; B stored
//   [k][n] has b_rows readable k rows (zeros beyond).
// KG = true (grouped along K, the token rows): group g sums rows seg_off[g] .. + seg_cnt[g]
//   of A and B (NULL: one group of K rows); C advances by c_gs per group; A stored [k][m]
//   has a_cols readable m columns (zeros beyond).
struct BwGemm {
    const uint16_t* A;
    long long lda, a_gs;
    const uint16_t* B;
    long long ldb, b_gs;
    float* C;
    long long ldc, c_gs;
    int M, N, K, a_cols, b_rows, groups;
    const int* seg_off;
    const int* seg_cnt;
    const int* tile_start;
};

template <bool A_K, bool B_K, bool KG, int BN, int BK, int NS>
__global__ void __launch_bounds__(kBwThreads) bw_gemm_kernel(const BwGemm p) {
    using TL = BwTile<BN, BK>;
    constexpr int WN = BN / 4, NI = WN / 8, NJ = WN / 16;   // warp tile columns, n8 tiles, x4 loads
    extern __shared__ __align__(128) uint16_t bw_smem[];
    __shared__ int s_g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int g = 0, m0, mvalid, kvalid_a, kvalid_b, KT;
    long long row0 = 0;
    if (!KG) {
        int tile = blockIdx.x;
        if (p.tile_start) {
            if (tid == 0) {
                int lo = 0, hi = p.groups;   // largest g with tile_start[g] <= tile
                if (tile >= p.tile_start[p.groups]) {
                    lo = -1;
                } else {
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (p.tile_start[mid] <= tile) lo = mid; else hi = mid;
                    }
                }
                s_g = lo;
            }
            __syncthreads();
            g = s_g;
            if (g < 0) return;
            tile -= p.tile_start[g];
        }
        row0 = p.seg_off ? p.seg_off[g] : 0;
        const int cnt = p.seg_cnt ? p.seg_cnt[g] : p.M;
        m0 = tile * kBwBM;
        mvalid = min(kBwBM, cnt - m0);
        if (mvalid <= 0) return;
        kvalid_a = p.K;
        kvalid_b = p.b_rows;
        KT = (p.K + BK - 1) / BK;
    } else {
        g = blockIdx.z;
        m0 = blockIdx.x * kBwBM;
        mvalid = min(kBwBM, p.M - m0);
        row0 = p.seg_off ? p.seg_off[g] : 0;
        kvalid_a = kvalid_b = p.seg_cnt ? p.seg_cnt[g] : p.K;
        KT = (kvalid_a + BK - 1) / BK;
    }
    const int n0 = blockIdx.y * BN;
    // operand origins: token rows are offset by row0 (along m for !KG, along k for KG)
    const uint16_t* Ag = KG ? p.A + row0 * p.lda : p.A + (row0 + m0) * p.lda;
    const uint16_t* Bg = KG ? p.B + row0 * p.ldb : p.B + (long long)g * p.b_gs;
    float* Cg = KG ? p.C + (long long)g * p.c_gs + (long long)m0 * p.ldc : p.C + (row0 + m0) * p.ldc;

    const uint32_t sbase = smem_u32(bw_smem);
    auto sA = [&](int st) { return sbase + (uint32_t)(st * (TL::A + TL::B)) * 2u; };
    auto sB = [&](int st) { return sbase + (uint32_t)(st * (TL::A + TL::B) + TL::A) * 2u; };

    auto load_stage = [&](int st, int kt) {
        const int k0 = kt * BK;
        constexpr int KC = BK / 8;   // 16-byte chunks along k
#pragma unroll
        for (int it = 0; it < kBwBM * BK / 8 / kBwThreads; ++it) {
            const int c = tid + it * kBwThreads;
            if (A_K) {   // 128 m rows x KC chunks of 8 k
                const int r = c / KC, col = (c % KC) * 8;
                const bool ok = r < mvalid && k0 + col < kvalid_a;
                const uint16_t* src = ok ? Ag + (long long)r * p.lda + k0 + col : p.A;
                cp_async16(sA(st) + (uint32_t)(r * TL::RowK + col) * 2u, src, ok);
            } else {     // BK k rows x 16 chunks of 8 m
                const int r = c >> 4, col = (c & 15) * 8;
                const bool ok = k0 + r < kvalid_a && m0 + col < p.a_cols;
                const uint16_t* src = ok ? Ag + (long long)(k0 + r) * p.lda + m0 + col : p.A;
                cp_async16(sA(st) + (uint32_t)(r * TL::RowM + col) * 2u, src, ok);
            }
        }
#pragma unroll
        for (int it = 0; it < BN * BK / 8 / kBwThreads; ++it) {
            const int c = tid + it * kBwThreads;
            if (B_K) {   // BN n rows x KC chunks of 8 k
                const int r = c / KC, col = (c % KC) * 8;
                const bool ok = n0 + r < p.N && k0 + col < p.K;
                const uint16_t* src = ok ? Bg + (long long)(n0 + r) * p.ldb + k0 + col : p.B;
                cp_async16(sB(st) + (uint32_t)(r * TL::RowK + col) * 2u, src, ok);
            } else {     // BK k rows x BN/8 chunks of 8 n
                const int r = c / (BN / 8), col = (c % (BN / 8)) * 8;
                const bool ok = k0 + r < kvalid_b && n0 + col < p.N;
                const uint16_t* src = ok ? Bg + (long long)(k0 + r) * p.ldb + n0 + col : p.B;
                cp_async16(sB(st) + (uint32_t)(r * TL::RowN + col) * 2u, src, ok);
            }
        }
    };

    float acc[4][NI][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NI; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[i][j][q] = 0.f;

    const int wm0 = (warp >> 2) * 64, wn0 = (warp & 3) * WN;
    const int li = lane >> 3, lr = lane & 7;
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) {
        if (s < KT) load_stage(s, s);
        cp_async_commit();
    }
    for (int kt = 0; kt < KT; ++kt) {
        cp_async_wait<NS - 2>();
        __syncthreads();
        const int nk = kt + NS - 1;
        if (nk < KT) load_stage(nk % NS, nk);
        cp_async_commit();
        const int st = kt % NS;
#pragma unroll
        for (int kk = 0; kk < BK; kk += 16) {
            uint32_t a[4][4], b[NJ][4];
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
                if (A_K) {
                    const int row = wm0 + mi * 16 + (lane & 15), col = kk + (lane >> 4) * 8;
                    ldmatrix_x4(sA(st) + (uint32_t)(row * TL::RowK + col) * 2u, a[mi][0], a[mi][1], a[mi][2], a[mi][3]);
                } else {
                    const int krow = kk + lr + (li >> 1) * 8, mcol = wm0 + mi * 16 + (li & 1) * 8;
                    ldmatrix_x4_trans(sA(st) + (uint32_t)(krow * TL::RowM + mcol) * 2u, a[mi][0], a[mi][1], a[mi][2],
                                      a[mi][3]);
                }
            }
#pragma unroll
            for (int nj = 0; nj < NJ; ++nj) {
                if (B_K) {
                    const int nrow = wn0 + nj * 16 + lr + (li >> 1) * 8, kcol = kk + (li & 1) * 8;
                    ldmatrix_x4(sB(st) + (uint32_t)(nrow * TL::RowK + kcol) * 2u, b[nj][0], b[nj][1], b[nj][2], b[nj][3]);
                } else {
                    const int krow = kk + lr + (li & 1) * 8, ncol = wn0 + nj * 16 + (li >> 1) * 8;
                    ldmatrix_x4_trans(sB(st) + (uint32_t)(krow * TL::RowN + ncol) * 2u, b[nj][0], b[nj][1], b[nj][2],
                                      b[nj][3]);
                }
            }
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                for (int ni = 0; ni < NI; ++ni)
                    mma_bf16_16816(acc[mi][ni], a[mi][0], a[mi][1], a[mi][2], a[mi][3], b[ni >> 1][(ni & 1) * 2],
                                   b[ni >> 1][(ni & 1) * 2 + 1]);
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni) {
            const int col = n0 + wn0 + ni * 8 + (lane & 3) * 2;
            if (col >= p.N) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = wm0 + mi * 16 + (lane >> 2) + h * 8;
                if (row < mvalid)
                    *reinterpret_cast<float2*>(Cg + (long long)row * p.ldc + col) =
                        make_float2(acc[mi][ni][2 * h], acc[mi][ni][2 * h + 1]);
            }
        }
}

// First 128-row tile of each group: tile_start[g] = sum_{g' < g} ceil(cnt[g'] / 128); and the
// S token slices of the router-weight gradient: slices[s] = floor(s T / S), slices[S + s] =
// its row count.
__global__ void bw_tile_table_kernel(const int* __restrict__ cnt, int groups, int* __restrict__ tile_start, int T,
                                     int S, int* __restrict__ slices) {
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int g = 0; g < groups; ++g) {
            tile_start[g] = acc;
            acc += (cnt[g] + kBwBM - 1) / kBwBM;
        }
        tile_start[groups] = acc;
        for (int q = 0; q < S; ++q) {
            const int a = (int)((long long)q * T / S), b = (int)((long long)(q + 1) * T / S);
            slices[q] = a;
            slices[S + q] = b - a;
        }
    }
}

// out[i] = sum_s part[s][i] in slice order (the router-weight gradient's K slices).
__global__ void bw_slice_sum_kernel(const float* __restrict__ part, int S, long long n, float* __restrict__ out) {
    for (long long i = 4 * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n;
         i += 4 * (long long)gridDim.x * blockDim.x) {
        float4 acc = *reinterpret_cast<const float4*>(part + i);
        for (int q = 1; q < S; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(part + (long long)q * n + i);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<float4*>(out + i) = acc;
    }
}

// Softmax statistics of one token's FP32 logits by one warp (lane L takes experts L, L + 32,
// ... in order, then a butterfly): row max and sum of exp(l - max).
__device__ __forceinline__ void bw_softmax_stats(const float* row, int E, float& m, float& s) {
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int e = lane; e < E; e += 32) mx = fmaxf(mx, row[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int e = lane; e < E; e += 32) sum += expf(row[e] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    m = mx;
    s = sum;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The given routing's weights, one warp per token: lane j < k holds slot j's probability
// p_j, the weight w_j (p_j / sum or p_j); valid = expert index in range.
__device__ __forceinline__ void bw_slot_weights(const float* lrow, const int32_t* irow, int E, int k, int norm,
                                                int& e, float& pj, float& wj, float& S) {
    const int lane = threadIdx.x & 31;
    float m, s;
    bw_softmax_stats(lrow, E, m, s);
    e = lane < k ? irow[lane] : -1;
    const bool ok = e >= 0 && e < E;
    pj = ok ? expf(lrow[e] - m) / s : 0.f;
    S = warp_sum(pj);
    wj = norm ? (S > 0.f ? pj / S : 0.f) : pj;
}

__global__ void bw_row_weight_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                                     const int32_t* __restrict__ slot_row, int T, int E, int k, int norm, int R,
                                     float* __restrict__ row_w) {
    const int lane = threadIdx.x & 31, nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int e;
        float pj, wj, S;
        bw_slot_weights(logits + (size_t)t * E, idx + (size_t)t * k, E, k, norm, e, pj, wj, S);
        if (lane < k) {
            const int r = slot_row[(size_t)t * k + lane];
            if (e >= 0 && e < E && r >= 0 && r < R) row_w[r] = wj;
        }
    }
}

// One warp per permuted row r (token t, weight w): from g, u (FP32, recomputed) and
// z = W_down^T dy:  h = silu(g) u -> bf16 H (the dW_down operand),  dw_row[r] = h . z (FP32,
// lanes in order then a butterfly),  dg, du -> bf16 dGU (gate first),  dO = bf16(w dy).
__global__ void bw_swiglu_kernel(const float* __restrict__ GU, const float* __restrict__ Z,
                                 const uint16_t* __restrict__ dYp, const float* __restrict__ row_w, int R, int D,
                                 int I, uint16_t* __restrict__ H, uint16_t* __restrict__ dGU,
                                 uint16_t* __restrict__ dO, float* __restrict__ dw_row) {
    const int lane = threadIdx.x & 31, nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < R; r += nwarps) {
        const float w = row_w[r];
        const float* gu = GU + (size_t)r * 2 * I;
        const float* z = Z + (size_t)r * I;
        float dws = 0.f;
        for (int i = 2 * lane; i < I; i += 64) {
            const float2 g2 = *reinterpret_cast<const float2*>(gu + i);
            const float2 u2 = *reinterpret_cast<const float2*>(gu + I + i);
            const float2 z2 = *reinterpret_cast<const float2*>(z + i);
            float hv[2], dg[2], du[2];
            const float gg[2] = {g2.x, g2.y}, uu[2] = {u2.x, u2.y}, zz[2] = {z2.x, z2.y};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float s = 1.f / (1.f + expf(-gg[q]));
                hv[q] = gg[q] * s * uu[q];
                dws += hv[q] * zz[q];
                const float dh = w * zz[q];
                dg[q] = dh * uu[q] * s * (1.f + gg[q] * (1.f - s));
                du[q] = dh * gg[q] * s;
            }
            *reinterpret_cast<uint32_t*>(H + (size_t)r * I + i) = pack_bf16x2(hv[0], hv[1]);
            *reinterpret_cast<uint32_t*>(dGU + (size_t)r * 2 * I + i) = pack_bf16x2(dg[0], dg[1]);
            *reinterpret_cast<uint32_t*>(dGU + (size_t)r * 2 * I + I + i) = pack_bf16x2(du[0], du[1]);
        }
        dws = warp_sum(dws);
        if (lane == 0) dw_row[r] = dws;
        const uint16_t* dy = dYp + (size_t)r * D;
        for (int d = 8 * lane; d < D; d += 256) {
            const uint4 v = *reinterpret_cast<const uint4*>(dy + d);
            uint4 o;
            o.x = pack_bf16x2(w * bf16_lo(v.x), w * bf16_hi(v.x));
            o.y = pack_bf16x2(w * bf16_lo(v.y), w * bf16_hi(v.y));
            o.z = pack_bf16x2(w * bf16_lo(v.z), w * bf16_hi(v.z));
            o.w = pack_bf16x2(w * bf16_lo(v.w), w * bf16_hi(v.w));
            *reinterpret_cast<uint4*>(dO + (size_t)r * D + d) = o;
        }
    }
}

// Routing backward, one warp per token: dw -> dp (through the renormalisation) -> dl
// (through the softmax), + the added logit gradient.  Writes dlogits [T, E] FP32, dl16
// [T, Epad] bf16 (zeros in the padding) and, when asked, dw [T, k].
__global__ void bw_route_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                                const int32_t* __restrict__ slot_row, const float* __restrict__ dw_row,
                                const float* __restrict__ dl_add, int T, int E, int k, int norm, int R, int Epad,
                                float* __restrict__ dlogits, uint16_t* __restrict__ dl16, float* __restrict__ dw_out) {
    const int lane = threadIdx.x & 31, nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* lrow = logits + (size_t)t * E;
        int e;
        float pj, wj, S;
        bw_slot_weights(lrow, idx + (size_t)t * k, E, k, norm, e, pj, wj, S);
        const bool ok = e >= 0 && e < E;
        float dwj = 0.f;
        if (ok) {
            const int r = slot_row[(size_t)t * k + lane];
            if (r >= 0 && r < R) dwj = dw_row[r];
        }
        if (dw_out && lane < k) dw_out[(size_t)t * k + lane] = dwj;
        const float sdw = warp_sum(dwj * wj);
        const float dpj = !ok ? 0.f : norm ? (S > 0.f ? (dwj - sdw) / S : 0.f) : dwj;
        const float pdp = warp_sum(pj * dpj);
        float m, s;
        bw_softmax_stats(lrow, E, m, s);
        for (int e0 = 0; e0 < Epad; e0 += 32) {
            const int ee = e0 + lane;
            float dpe = 0.f;
            for (int j = 0; j < k; ++j) {   // slot order
                const int ej = __shfl_sync(0xffffffffu, ok ? e : -1, j);
                const float dj = __shfl_sync(0xffffffffu, dpj, j);
                if (ej == ee) dpe += dj;
            }
            if (ee < E) {
                const float p = expf(lrow[ee] - m) / s;
                float dl = p * (dpe - pdp);
                if (dl_add) dl += dl_add[(size_t)t * E + ee];
                dlogits[(size_t)t * E + ee] = dl;
                dl16[(size_t)t * Epad + ee] = to_bf16_bits(dl);
            } else if (ee < Epad) {
                dl16[(size_t)t * Epad + ee] = 0;
            }
        }
    }
}

// db[e] = sum_t dl[t, e]: one block; R = 512 / E threads per expert add rows r, r + R, ... in
// order, then thread e adds the R partial sums in order.
__global__ void __launch_bounds__(512) bw_colsum_kernel(const float* __restrict__ dl, int T, int E,
                                                        float* __restrict__ db) {
    __shared__ float s_part[512];
    const int Rr = 512 / E;
    if (threadIdx.x < Rr * E) {
        const int e = threadIdx.x % E, r = threadIdx.x / E;
        float acc = 0.f;
        for (int t = r; t < T; t += Rr) acc += dl[(size_t)t * E + e];
        s_part[threadIdx.x] = acc;
    }
    __syncthreads();
    if (threadIdx.x < E) {
        float acc = 0.f;
        for (int r = 0; r < Rr; ++r) acc += s_part[r * E + threadIdx.x];
        db[threadIdx.x] = acc;
    }
}

// dx[t] = sum_j dXr[slot_row[t, j]] (slot order) + dxr[t] (+ dy[t]), four features per thread.
__global__ void bw_dx_kernel(const float* __restrict__ dXr, const int32_t* __restrict__ slot_row,
                             const float* __restrict__ dxr, const uint16_t* __restrict__ dy, int T, int D, int k,
                             int R, int residual, float* __restrict__ dx) {
    const int q = D / 4;
    const long long n = (long long)T * q;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(i / q), d = (int)(i % q) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int r = slot_row[(size_t)t * k + j];
            if (r < 0 || r >= R) continue;
            const float4 v = *reinterpret_cast<const float4*>(dXr + (size_t)r * D + d);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        const float4 v = *reinterpret_cast<const float4*>(dxr + (size_t)t * D + d);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        if (residual) {
            const uint2 y = *reinterpret_cast<const uint2*>(dy + (size_t)t * D + d);
            acc.x += bf16_lo(y.x); acc.y += bf16_hi(y.x); acc.z += bf16_lo(y.y); acc.w += bf16_hi(y.y);
        }
        *reinterpret_cast<float4*>(dx + (size_t)t * D + d) = acc;
    }
}

}  // namespace moe

using namespace moe;

namespace {

// Workspace of moe_backward: the forward's workspace (router and permutation scratch, and
// the device error word at its start), then the backward's own buffers.  R = T k rows.
struct BwPlan {
    size_t sub, sub_bytes, logits, idx, w, counts, offsets, tiles, slices, row_token, slot_row, row_w, dw_row, xp, dyp,
        gu, z, h, dgu, dout, dxr_rows, dlog, dl16, dxr, dwr_part, total;
    int R, Epad, S;
};

// Token slices of the router-weight gradient dW_r = dl^T x (its K is T): one per 512 tokens,
// at most 16, a function of T only (so the summation order does not depend on the GPU).
inline int bw_router_slices(int T) { return std::max(1, std::min(16, T / 512)); }

size_t bw_align(size_t v) { return (v + 255) / 256 * 256; }

BwPlan bw_plan(const moe_dims& d, size_t sub_bytes) {
    BwPlan p;
    p.R = d.T * d.k;
    p.Epad = (d.E + 7) / 8 * 8;
    p.S = bw_router_slices(d.T);
    const size_t T = d.T, D = d.D, E = d.E, k = d.k, I = d.I, R = p.R;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = bw_align(off + bytes);
        return at;
    };
    p.sub = take(sub_bytes);
    p.sub_bytes = sub_bytes;
    p.logits = take(T * E * 4);
    p.idx = take(T * k * 4);
    p.w = take(T * k * 4);
    p.counts = take(E * 4);
    p.offsets = take((E + 1) * 4);
    p.tiles = take((E + 1) * 4);
    p.slices = take((size_t)2 * p.S * 4);
    p.row_token = take(R * 4);
    p.slot_row = take(R * 4);
    p.row_w = take(R * 4);
    p.dw_row = take(R * 4);
    p.xp = take(R * D * 2);
    p.dyp = take(R * D * 2);
    p.gu = take(R * 2 * I * 4);
    p.z = take(R * I * 4);
    p.h = take(R * I * 2);
    p.dgu = take(R * 2 * I * 2);
    p.dout = take(R * D * 2);
    p.dxr_rows = take(R * D * 4);
    p.dlog = take(T * E * 4);
    p.dl16 = take(T * p.Epad * 2);
    p.dxr = take(T * D * 4);
    p.dwr_part = take(p.S > 1 ? (size_t)p.S * E * D * 4 : 0);
    p.total = off;
    return p;
}

moe_dims bw_dims(const moe_dims* d) {
    moe_dims f = *d;
    f.tile_m = 1;
    return f;
}

bool bw_aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

template <bool A_K, bool B_K, bool KG>
cudaError_t bw_gemm(const BwGemm& g, int grid_x, int grid_z, cudaStream_t s) {
    auto kern = bw_gemm_kernel<A_K, B_K, KG, kBwBN, kBwBK, kBwStages>;
    constexpr int smem = bw_smem_bytes<kBwBN, kBwBK, kBwStages>();
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    if (grid_x < 1 || grid_z < 1) return cudaSuccess;
    return launch_kernel(kern, dim3(grid_x, (g.N + kBwBN - 1) / kBwBN, grid_z), dim3(kBwThreads), smem, s, false, g);
}

}  // namespace

extern "C" size_t moe_backward_workspace_size(const moe_dims* dims) {
    if (!dims) return 0;
    const moe_dims f = bw_dims(dims);
    const size_t sub = moe_workspace_size(&f, nullptr);
    if (sub == 0) return 0;
    return bw_plan(f, sub).total;
}

extern "C" moe_status moe_backward(const moe_bf16* x, const moe_bf16* W_r, const float* bias, const moe_bf16* W_gate_up,
                                   const moe_bf16* W_down, const moe_bf16* dy, const int32_t* topk_idx,
                                   const float* dlogits_add, int residual, const moe_dims* dims, float* dx,
                                   float* dW_r, float* dbias, float* dW_gate_up, float* dW_down, float* dlogits,
                                   float* dw, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!dims) return MOE_ERR_INVALID_ARG;
    const moe_dims f = bw_dims(dims);
    const size_t sub = moe_workspace_size(&f, nullptr);
    if (sub == 0) {
        if (f.T < 1 || f.D < 1 || f.E < 1 || f.k < 1 || f.I < 1 || (f.norm_topk_prob != 0 && f.norm_topk_prob != 1))
            return MOE_ERR_INVALID_ARG;
        return MOE_ERR_UNSUPPORTED;
    }
    if (residual != 0 && residual != 1) return MOE_ERR_INVALID_ARG;
    if (!x || !W_r || !W_gate_up || !W_down || !dy || !topk_idx || !dx || !dW_r || !dW_gate_up || !dW_down || !ws)
        return MOE_ERR_INVALID_ARG;
    const void* p16[] = {x, W_r, W_gate_up, W_down, dy, dx, dW_r, dW_gate_up, dW_down};
    for (const void* q : p16)
        if (!bw_aligned(q, 16)) return MOE_ERR_INVALID_ARG;
    const void* p4[] = {bias, topk_idx, dlogits_add, dbias, dlogits, dw};
    for (const void* q : p4)
        if (q && !bw_aligned(q, 4)) return MOE_ERR_INVALID_ARG;
    if (!bw_aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    const BwPlan P = bw_plan(f, sub);
    if (ws_bytes < P.total) return MOE_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    auto F = [&](size_t at) { return reinterpret_cast<float*>(w + at); };
    auto Iw = [&](size_t at) { return reinterpret_cast<int32_t*>(w + at); };
    auto H = [&](size_t at) { return reinterpret_cast<uint16_t*>(w + at); };
    const int T = f.T, D = f.D, E = f.E, k = f.k, I = f.I, R = P.R, norm = f.norm_topk_prob;
    const uint16_t* x16 = reinterpret_cast<const uint16_t*>(x);
    const uint16_t* wr16 = reinterpret_cast<const uint16_t*>(W_r);
    const uint16_t* wgu16 = reinterpret_cast<const uint16_t*>(W_gate_up);
    const uint16_t* wdn16 = reinterpret_cast<const uint16_t*>(W_down);
    const uint16_t* dy16 = reinterpret_cast<const uint16_t*>(dy);
    float* logits = F(P.logits);
    float* dlog = dlogits ? dlogits : F(P.dlog);
    int32_t *counts = Iw(P.counts), *offsets = Iw(P.offsets), *tiles = Iw(P.tiles);
    int32_t *row_token = Iw(P.row_token), *slot_row = Iw(P.slot_row);

    // the forward's FP32 logits (its own selection is not used), the given routing's permutation
    moe_status st = moe_route(x, W_r, bias, &f, logits, Iw(P.idx), F(P.w), w + P.sub, P.sub_bytes, stream);
    if (st != MOE_OK) return st;
    st = moe_permute(topk_idx, nullptr, x, &f, counts, offsets, row_token, slot_row, nullptr,
                     reinterpret_cast<moe_bf16*>(w + P.xp), R, w + P.sub, P.sub_bytes, stream);
    if (st != MOE_OK) return st;

    cudaError_t e = launch_gather_rows(dy16, row_token, R, D, H(P.dyp), false, s);
    const int sms = device_sm_count();
    const int wblocks = sms * 8;   // warp-per-item kernels: 8 warps per block
    int32_t* slices = Iw(P.slices);
    if (e == cudaSuccess)
        e = launch_kernel(bw_tile_table_kernel, dim3(1), dim3(32), 0, s, false, (const int*)counts, E, tiles, T, P.S,
                          slices);
    if (e == cudaSuccess)
        e = launch_kernel(bw_row_weight_kernel, dim3(std::min(wblocks, (T + 7) / 8)), dim3(256), 0, s, false,
                          (const float*)logits, topk_idx, (const int32_t*)slot_row, T, E, k, norm, R, F(P.row_w));
    const int mtiles = (R + kBwBM - 1) / kBwBM + E;   // bound on sum_e ceil(count_e / 128)
    // g, u = W_gate_up[e] x   (rows grouped by expert)
    if (e == cudaSuccess) {
        BwGemm g{H(P.xp), D, 0, wgu16, D, (long long)2 * I * D, F(P.gu), 2 * I, 0, 0, 2 * I, D, 0, 0, E,
                 offsets, counts, tiles};
        e = bw_gemm<true, true, false>(g, mtiles, 1, s);
    }
    // z = W_down[e]^T dy
    if (e == cudaSuccess) {
        BwGemm g{H(P.dyp), D, 0, wdn16, I, (long long)D * I, F(P.z), I, 0, 0, I, D, 0, D, E, offsets, counts, tiles};
        e = bw_gemm<true, false, false>(g, mtiles, 1, s);
    }
    if (e == cudaSuccess)
        e = launch_kernel(bw_swiglu_kernel, dim3(std::min(wblocks, (R + 7) / 8)), dim3(256), 0, s, false,
                          (const float*)F(P.gu), (const float*)F(P.z), (const uint16_t*)H(P.dyp),
                          (const float*)F(P.row_w), R, D, I, H(P.h), H(P.dgu), H(P.dout), F(P.dw_row));
    // dW_down[e] = sum over e's rows of (w dy) h^T
    if (e == cudaSuccess) {
        BwGemm g{H(P.dout), D, 0, H(P.h), I, 0, dW_down, I, (long long)D * I, D, I, 0, D, 0, E, offsets, counts, nullptr};
        e = bw_gemm<false, false, true>(g, (D + kBwBM - 1) / kBwBM, E, s);
    }
    // dX rows = [dg du] W_gate_up[e]
    if (e == cudaSuccess) {
        BwGemm g{H(P.dgu), 2 * I, 0, wgu16, D, (long long)2 * I * D, F(P.dxr_rows), D, 0, 0, D, 2 * I, 0, 2 * I, E,
                 offsets, counts, tiles};
        e = bw_gemm<true, false, false>(g, mtiles, 1, s);
    }
    // dW_gate_up[e] = sum over e's rows of [dg du] x^T
    if (e == cudaSuccess) {
        BwGemm g{H(P.dgu), 2 * I, 0, H(P.xp), D, 0, dW_gate_up, D, (long long)2 * I * D, 2 * I, D, 0, 2 * I, 0, E,
                 offsets, counts, nullptr};
        e = bw_gemm<false, false, true>(g, (2 * I + kBwBM - 1) / kBwBM, E, s);
    }
    // routing: dw -> dl
    if (e == cudaSuccess)
        e = launch_kernel(bw_route_kernel, dim3(std::min(wblocks, (T + 7) / 8)), dim3(256), 0, s, false,
                          (const float*)logits, topk_idx, (const int32_t*)slot_row, (const float*)F(P.dw_row),
                          dlogits_add, T, E, k, norm, R, P.Epad, dlog, H(P.dl16), dw);
    // dW_r = dl^T x: S token slices as K groups, then their sum in slice order
    if (e == cudaSuccess) {
        float* dst = P.S > 1 ? F(P.dwr_part) : dW_r;
        BwGemm g{H(P.dl16), P.Epad, 0, x16, D, 0, dst, D, (long long)E * D, E, D, T, P.Epad, 0, P.S, slices,
                 slices + P.S, nullptr};
        e = bw_gemm<false, false, true>(g, (E + kBwBM - 1) / kBwBM, P.S, s);
        if (e == cudaSuccess && P.S > 1) {
            const long long n = (long long)E * D;
            const int blocks = (int)std::min<long long>((n / 4 + 255) / 256, (long long)sms * 8);
            e = launch_kernel(bw_slice_sum_kernel, dim3(blocks), dim3(256), 0, s, false, (const float*)F(P.dwr_part),
                              P.S, n, dW_r);
        }
    }
    // dx (router part) = dl W_r
    if (e == cudaSuccess) {
        BwGemm g{H(P.dl16), P.Epad, 0, wr16, D, 0, F(P.dxr), D, 0, T, D, P.Epad, 0, E, 1, nullptr, nullptr, nullptr};
        e = bw_gemm<true, false, false>(g, (T + kBwBM - 1) / kBwBM, 1, s);
    }
    if (e == cudaSuccess && dbias)
        e = launch_kernel(bw_colsum_kernel, dim3(1), dim3(512), 0, s, false, (const float*)dlog, T, E, dbias);
    if (e == cudaSuccess) {
        const long long n = (long long)T * (D / 4);
        const int blocks = (int)std::min<long long>((n + 255) / 256, (long long)sms * 16);
        e = launch_kernel(bw_dx_kernel, dim3(blocks), dim3(256), 0, s, false, (const float*)F(P.dxr_rows),
                          (const int32_t*)slot_row, (const float*)F(P.dxr), dy16, T, D, k, R, residual, dx);
    }
    if (e != cudaSuccess) {
        note_cuda_error((int)e);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}
