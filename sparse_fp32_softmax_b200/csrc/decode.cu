// decode.cu -- the MoE block for one token (a batch-1 decode step) in one persistent kernel.
//
// "27. Mixture of experts" (inference.shantanugoel.com): section "The router" (logits,
// FP32 softmax, top-k with index tie-break, renormalisation, y = sum_i w_i expert_i(x)) and
// section "Dispatch" (gate_up [E, 2I, D], down [E, D, I], expert(x) = down(silu(gate x) *
// up x)); section "The economics of MoE inference": a decode step is bound by reading the
// weights of the experts its token chose, so everything else has to hide under that read.
//
// For one token the chain of separate kernels (router, selection + permutation, gate_up,
// down, combine) costs more in launches and dependency waits than the weights take to
// stream, and the tensor-core tiles (128 weight rows x 64 tokens) hold one useful column.
// Here one block per SM runs the whole block:
//   1. router: block b computes the logits of experts b, b + G, ... (8 warps, one D slice
//      each, slices added in slice order: the order of the small-T router) and stores each
//      with a ready flag in one 64-bit word of the workspace;
//   2. selection: every block polls the E words until all are flagged and selects the
//      token's k experts (one warp, the same code and inputs as the selection kernel, so the
//      same result); slot j is expert idx[j];
//   3. gate_up: the (slot, feature) pairs are split evenly over the blocks; 8 warps load each
//      pair's gate row and up row into registers and compute h = silu(gate . x) * (up . x),
//      rounded to bf16, into the workspace.  Meanwhile a copy warp streams the block's down
//      rows into a ring of shared-memory stages (bulk copies completing on mbarriers), so
//      they are there when h is;  grid barrier;
//   4. down + combine: block b owns output rows [b*D/G, (b+1)*D/G) of every slot; it reads
//      h into shared memory, multiplies the down rows in the ring by h with warp MMAs, and adds
//      the k weighted expert outputs in slot order (FP32), then the residual, and rounds once
//      to bf16 -- no permutation, no FP32 slot buffer, no combine kernel.
// Every wait is bounded (kErrWaitGrid, kErrWaitProducer, kErrWaitMma, kErrWaitTail).
// The workspace words the kernel waits on (flagged logits, barrier counter) are zeroed by
// the host before each launch.
#include "common.cuh"
#include "select.cuh"

namespace moe {

namespace {

// Dot product of 8 bf16 weights with x values taken from the two FP32 planes, one chain
// (the router's order).
__device__ __forceinline__ float dot8(const uint4& w, const float4& lo, const float4& hi, float acc) {
    acc = fmaf(bf16_lo(w.x), lo.x, acc);
    acc = fmaf(bf16_hi(w.x), lo.y, acc);
    acc = fmaf(bf16_lo(w.y), lo.z, acc);
    acc = fmaf(bf16_hi(w.y), lo.w, acc);
    acc = fmaf(bf16_lo(w.z), hi.x, acc);
    acc = fmaf(bf16_hi(w.z), hi.y, acc);
    acc = fmaf(bf16_lo(w.w), hi.z, acc);
    acc = fmaf(bf16_hi(w.w), hi.w, acc);
    return acc;
}

// The same as two half sums (values 0-3 into acc0, 4-7 into acc1): shorter FMA chains.
__device__ __forceinline__ void dot8_2(const uint4& w, const float4& lo, const float4& hi, float& acc0, float& acc1) {
    acc0 = fmaf(bf16_lo(w.x), lo.x, acc0);
    acc1 = fmaf(bf16_lo(w.z), hi.x, acc1);
    acc0 = fmaf(bf16_hi(w.x), lo.y, acc0);
    acc1 = fmaf(bf16_hi(w.z), hi.y, acc1);
    acc0 = fmaf(bf16_lo(w.y), lo.z, acc0);
    acc1 = fmaf(bf16_lo(w.w), hi.z, acc1);
    acc0 = fmaf(bf16_hi(w.y), lo.w, acc0);
    acc1 = fmaf(bf16_hi(w.w), hi.w, acc1);
}

// Two E4M3 values (bytes 0 and 1 of `two`) as FP32, exactly (E4M3 -> fp16 -> FP32).
__device__ __forceinline__ float2 e4m3x2_float2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Dot product of 16 E4M3 weights (byte i = value i) with 16 x values from the two FP32
// planes (pieces 2c and 2c + 1), as two half sums.
__device__ __forceinline__ void dot16_e4m3(const uint4& w, const float4& lo0, const float4& hi0, const float4& lo1,
                                           const float4& hi1, float& acc0, float& acc1) {
    float2 a = e4m3x2_float2(w.x), bq = e4m3x2_float2(w.x >> 16);
    acc0 = fmaf(a.x, lo0.x, acc0); acc0 = fmaf(a.y, lo0.y, acc0);
    acc0 = fmaf(bq.x, lo0.z, acc0); acc0 = fmaf(bq.y, lo0.w, acc0);
    a = e4m3x2_float2(w.y); bq = e4m3x2_float2(w.y >> 16);
    acc1 = fmaf(a.x, hi0.x, acc1); acc1 = fmaf(a.y, hi0.y, acc1);
    acc1 = fmaf(bq.x, hi0.z, acc1); acc1 = fmaf(bq.y, hi0.w, acc1);
    a = e4m3x2_float2(w.z); bq = e4m3x2_float2(w.z >> 16);
    acc0 = fmaf(a.x, lo1.x, acc0); acc0 = fmaf(a.y, lo1.y, acc0);
    acc0 = fmaf(bq.x, lo1.z, acc0); acc0 = fmaf(bq.y, lo1.w, acc0);
    a = e4m3x2_float2(w.w); bq = e4m3x2_float2(w.w >> 16);
    acc1 = fmaf(a.x, hi1.x, acc1); acc1 = fmaf(a.y, hi1.y, acc1);
    acc1 = fmaf(bq.x, hi1.z, acc1); acc1 = fmaf(bq.y, hi1.w, acc1);
}

// Dot product of 16 E4M3 weights with 16 bf16 values (h0: values 0-7, h1: values 8-15), as
// two half sums.
__device__ __forceinline__ void dot16_e4m3_bf16(const uint4& w, const uint4& h0, const uint4& h1, float& acc0,
                                                float& acc1) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    const uint32_t hh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 a = e4m3x2_float2(ww[q]), bq = e4m3x2_float2(ww[q] >> 16);
        float& acc = (q & 1) ? acc1 : acc0;
        acc = fmaf(a.x, bf16_lo(hh[2 * q]), acc);
        acc = fmaf(a.y, bf16_hi(hh[2 * q]), acc);
        acc = fmaf(bq.x, bf16_lo(hh[2 * q + 1]), acc);
        acc = fmaf(bq.y, bf16_hi(hh[2 * q + 1]), acc);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int kRouterGroup = 4;   // experts whose router rows one block loads together

}  // namespace

// VPL: logits per lane in the selection (E <= 32 * VPL); F8: E4M3 expert weights with FP32
// row scales (applied to the FP32 sums) instead of bf16.
template <int VPL, bool F8>
__global__ void __launch_bounds__(kDecThreads, 1) decode_block_kernel(const DecodeArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ int s_idx[kMaxK];
    __shared__ float s_w[kMaxK];
    __shared__ float s_rpart[kDecWarps][kRouterGroup];
    __shared__ int s_nsel;   // slots published by the selection

    const int D = a.D, E = a.E, k = a.k, I = a.I;
    const int G = gridDim.x, b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = a.stages;
    const int nd_max = (D + G - 1) / G;
    const DecodeLayout L = decode_layout(D, k, I, nd_max, NS, F8);
    uint8_t* ring = smem + L.ring;
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    uint16_t* hs = reinterpret_cast<uint16_t*>(smem + L.hs);
    float* val = reinterpret_cast<float*>(smem + L.val);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + NS;
    const int DC = D / 8;   // 16-byte pieces of a row of D bf16 values
    const float4* xlo = reinterpret_cast<const float4*>(xs);
    const float4* xhi = reinterpret_cast<const float4*>(xs + D / 2);

    if (threadIdx.x < kMaxK) s_idx[threadIdx.x] = 0;   // in range until the selection publishes
    if (threadIdx.x == 0) {
        s_nsel = 0;
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_fence_init();
    }
    // nothing before this point reads the caller's tensors or the workspace
    pdl_wait();

    // x as FP32: piece c (values 8c..8c+7) is float4 c of the low plane (values 8c..8c+3)
    // and float4 c of the high plane (8c+4..8c+7)
    for (int c = threadIdx.x; c < DC; c += blockDim.x) {
        const uint4 v = ld_v4(a.x + (size_t)c * 8);
        reinterpret_cast<float4*>(xs)[c] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
        reinterpret_cast<float4*>(xs + D / 2)[c] =
            make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
    __syncthreads();

    // ---- 1. router logits of experts b, b + G, ...: warp w sums slice w of D (D/8 values;
    // lane L takes its pieces L, L + 32 in order), the 8 slice sums are added in slice order
    if (warp >= 1) {
        const int cw = warp - 1;
        const int per = D / 64;   // pieces per slice
        for (int e0 = b; e0 < E; e0 += kRouterGroup * G) {
            uint4 wv[kRouterGroup][2];
#pragma unroll
            for (int q = 0; q < kRouterGroup; ++q)
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int e = e0 + q * G, c = lane + 32 * m;
                    wv[q][m] = (e < E && c < per)
                                   ? ld_stream_v4(a.W_r + (size_t)e * D + (size_t)(cw * per + c) * 8)
                                   : make_uint4(0u, 0u, 0u, 0u);
                }
            float acc[kRouterGroup] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int c = lane + 32 * m;
                if (c < per) {
                    const int cc = cw * per + c;
#pragma unroll
                    for (int q = 0; q < kRouterGroup; ++q) acc[q] = dot8(wv[q][m], xlo[cc], xhi[cc], acc[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < kRouterGroup; ++q) {
                const float v = warp_sum(acc[q]);
                if (lane == 0) s_rpart[cw][q] = v;
            }
            named_barrier_sync(1, kDecWarps * 32);
            if (cw == 0 && lane < kRouterGroup && e0 + lane * G < E) {
                float v = s_rpart[0][lane];
#pragma unroll
                for (int w = 1; w < kDecWarps; ++w) v += s_rpart[w][lane];
                // the logit with a ready flag in one 64-bit store: readers poll the word itself
                st_relaxed_gpu_u64(a.lgf + e0 + lane * G, (1ull << 32) | __float_as_uint(v));
            }
            named_barrier_sync(1, kDecWarps * 32);
        }
    }

    const int d0 = (int)((long long)D * b / G), d1 = (int)((long long)D * (b + 1) / G);
    const int nd = d1 - d0;                                  // output rows of this block
    const int ND = nd > 0 ? k : 0;                           // down stages: one per slot

    if (warp == 0) {
        // ---- 2. the copy warp selects.  It polls the E flagged logits (written by the router
        // blocks of this launch, zero before it) and ranks them with the arithmetic of the
        // selection kernel (select.cuh: order-preserving keys, -0.0 = +0.0, the lower index
        // first among equal keys), so the result is the same.  After each round it publishes
        // the slot's expert (s_idx[j], then s_nsel = j + 1) and starts the copy of that
        // expert's down rows: the compute warps start on slot 0 while later rounds run.  The
        // softmax weights are finished after the rounds (only the combine needs them).
        const uint64_t t0 = globaltimer_ns();
        float v[VPL];
        uint32_t key[VPL];
        uint32_t kmax = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            key[i] = 0u;   // below every finite logit's key
            v[i] = 0.f;
            if (e < E) {
                unsigned long long w = ld_relaxed_gpu_u64(a.lgf + e);
                while ((w >> 32) == 0ull) {
                    if (globaltimer_ns() - t0 > a.wait_ns) {
                        set_error(a.err, kErrWaitGrid);
                        break;
                    }
                    w = ld_relaxed_gpu_u64(a.lgf + e);
                }
                v[i] = __uint_as_float((uint32_t)w);
                if (a.bias) v[i] = v[i] + __ldg(a.bias + e);
                if (b == 0 && a.logits_out) a.logits_out[e] = v[i];
                v[i] = v[i] + 0.0f;
                key[i] = float_order_key(v[i]);
                kmax = key[i] > kmax ? key[i] : kmax;
            }
        }
        const float mx = float_from_order_key(__reduce_max_sync(0xffffffffu, kmax));
        const uint32_t bytes = (uint32_t)nd * I * (F8 ? 1 : 2);   // rows d0..d1-1 of an expert: contiguous
        int my_e = 0;
        float my_l = 0.f;
        for (int j = 0; j < k; ++j) {
            uint32_t bk = 0;
            int bi = 0;
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (key[i] > bk) {   // strict: the lane's lowest index among equal keys
                    bk = key[i];
                    bi = i;
                }
            const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t cand = (bk == mk && bk != 0u) ? 0xFFFFFFFFu - (uint32_t)(lane + 32 * bi) : 0u;
            int e = (int)(0xFFFFFFFFu - __reduce_max_sync(0xffffffffu, cand));
            if ((e & 31) == lane) {
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    if (i == (e >> 5)) key[i] = 0u;
            }
            if (lane == j) {
                my_e = e;
                my_l = float_from_order_key(mk);
            }
            if (e < 0 || e >= E) {   // cannot happen for finite logits
                if (lane == 0) set_error(a.err, kErrBadIndex);
                e = 0;
            }
            if (lane == 0) {
                s_idx[j] = e;
                __threadfence_block();
                *reinterpret_cast<volatile int*>(&s_nsel) = j + 1;
            }
            if (j < NS && nd > 0) {   // the first round of ring slot j: no wait for a free slot
                if (lane == 0) mbar_arrive_expect_tx(full + j, bytes);
                __syncwarp();
                if constexpr (F8) {   // packed rows: one copy
                    if (lane == 0) bulk_load(ring + (size_t)j * L.sb, a.W_dn8 + ((size_t)e * D + d0) * I, bytes, full + j);
                } else {
                    const uint16_t* src = a.W_dn + ((size_t)e * D + d0) * I;
                    for (int rr = lane; rr < nd; rr += 32)   // one copy per row: the padded stride
                        bulk_load(ring + (size_t)j * L.sb + (size_t)rr * L.rs, src + (size_t)rr * I,
                                  (uint32_t)I * 2, full + j);
                }
            }
        }
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (lane + 32 * i < E) sum += expf(v[i] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float pr = (lane < k) ? expf(my_l - mx) / sum : 0.f;   // FP32 softmax probability
        float wv = pr;
        if (a.norm) {
            float tot = pr;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
            wv = pr / tot;
        }
        if (lane < k) {
            s_w[lane] = wv;
            if (b == 0) {
                a.idx_out[lane] = my_e;
                a.w_out[lane] = wv;
            }
        }
        __syncwarp();
        // the down rows that find no free ring slot before the down phase: into L2 now, into
        // the ring as the compute warps free slots
        if (lane == 0) {
            for (int j = NS; j < ND; ++j)
                bulk_prefetch_l2(F8 ? (const void*)(a.W_dn8 + ((size_t)s_idx[j] * D + d0) * I)
                                    : (const void*)(a.W_dn + ((size_t)s_idx[j] * D + d0) * I),
                                 bytes);
            int issued = ND < NS ? ND : NS, s = 0, r = 1;    // slot s of round r
            for (int i = NS; i < ND; ++i) {
                if (!mbar_wait(empty + s, (r - 1) & 1, a.err, kErrWaitProducer, a.wait_ns)) break;
                mbar_arrive_expect_tx(full + s, bytes);
                if constexpr (F8) {
                    bulk_load(ring + (size_t)s * L.sb, a.W_dn8 + ((size_t)s_idx[i] * D + d0) * I, bytes, full + s);
                } else {
                    const uint16_t* src = a.W_dn + ((size_t)s_idx[i] * D + d0) * I;
                    for (int rr = 0; rr < nd; ++rr)
                        bulk_load(ring + (size_t)s * L.sb + (size_t)rr * L.rs, src + (size_t)rr * I, (uint32_t)I * 2,
                                  full + s);
                }
                issued = i + 1;
                if (++s == NS) {
                    s = 0;
                    ++r;
                }
            }
            // no copy may still be writing into shared memory when the block exits
            for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
                mbar_wait(full + i % NS, (i / NS) & 1, a.err, kErrWaitTail, a.wait_ns);
        }
        __syncwarp();
        named_barrier_sync(2, kDecThreads);   // the combine reads s_w
        return;
    }

    const int cw = warp - 1;
    const int ct = threadIdx.x - 32;
    // ---- 3. gate_up.  The block's pairs, slot-major: for slot j the features
    // [floor(I(bk+j)/(Gk)), floor(I((b+1)k+j)/(Gk))) taken mod I -- a share of every slot, the
    // boundaries shifted by j/k of a block from slot to slot so that block totals stay within a
    // few pairs of each other -- so every block starts on slot 0 while the selection goes on.  Warp cw takes the block's pairs cw, cw + 8, ...  Its lanes
    // load the pair's gate row and up row straight into registers (16-byte pieces lane,
    // lane + 32, ...: the loads of a warp cover whole rows), the next pair's loads in flight
    // while the current pair is computed.  (Measured on B200: the copy engine of one SM streams
    // about 30 GB/s of 4-8 KB bulk copies, below the SM's share of HBM; the load units of 8
    // warps with two pairs each in flight do better, and leave the copy engine to the down rows.)
    {
        int qj = 0, qf = 0, qfe = 0;   // the warp's next pair: slot qj, feature qf (range end qfe)
        auto slot_range = [&](int j) {   // unwrapped feature range; feature = value mod I
            qf = (int)((long long)I * (b * k + j) / ((long long)G * k));
            qfe = (int)((long long)I * ((b + 1) * k + j) / ((long long)G * k));
        };
        auto advance = [&](int n) {
            qf += n;
            while (qj < k && qf >= qfe) {
                const int over = qf - qfe;
                if (++qj < k) {
                    slot_range(qj);
                    qf += over;
                }
            }
        };
        slot_range(0);
        advance(cw);
        // 16-byte pieces of a gate/up row per lane (a bf16 piece is 8 values, an E4M3 piece 16)
        constexpr int NCH = F8 ? kDecChunks8 : kDecChunks;
        const int RC = F8 ? D / 16 : DC;   // pieces of a row
        uint4 ga[NCH], ua[NCH], gb[NCH], ub[NCH];
        auto load_pair = [&](int j, int f, uint4 (&g)[NCH], uint4 (&v)[NCH]) {
            // slot j's expert is published by the copy warp's selection round j
            if (*reinterpret_cast<volatile int*>(&s_nsel) <= j) {
                const uint64_t t0 = globaltimer_ns();
                while (*reinterpret_cast<volatile int*>(&s_nsel) <= j)
                    if (globaltimer_ns() - t0 > a.wait_ns) {
                        set_error(a.err, kErrWaitMma);
                        break;
                    }
            }
            const int e = *reinterpret_cast<volatile int*>(&s_idx[j]);
            if constexpr (F8) {   // the gate row; the up row is I rows on
                const uint8_t* gr = a.W_gu8 + ((size_t)e * 2 * I + f) * D;
                const uint8_t* ur = gr + (size_t)I * D;
#pragma unroll
                for (int m = 0; m < NCH; ++m) {
                    const int c = lane + 32 * m;
                    if (c < RC) {
                        g[m] = ld_stream_v4(gr + (size_t)c * 16);
                        v[m] = ld_stream_v4(ur + (size_t)c * 16);
                    }
                }
            } else {
                const uint16_t* gr = a.W_gu + ((size_t)e * 2 * I + f) * D;
                const uint16_t* ur = gr + (size_t)I * D;
#pragma unroll
                for (int m = 0; m < NCH; ++m) {
                    const int c = lane + 32 * m;
                    if (c < RC) {
                        g[m] = ld_stream_v4(gr + (size_t)c * 8);
                        v[m] = ld_stream_v4(ur + (size_t)c * 8);
                    }
                }
            }
        };
        auto finish_pair = [&](int j, int f, const uint4 (&g)[NCH], const uint4 (&v)[NCH]) {
            float ag0 = 0.f, ag1 = 0.f, au0 = 0.f, au1 = 0.f;
#pragma unroll
            for (int m = 0; m < NCH; ++m) {
                const int c = lane + 32 * m;
                if (c < RC) {
                    if constexpr (F8) {   // values 16c..16c+15: x pieces 2c and 2c + 1
                        const float4 lo0 = xlo[2 * c], hi0 = xhi[2 * c], lo1 = xlo[2 * c + 1], hi1 = xhi[2 * c + 1];
                        dot16_e4m3(g[m], lo0, hi0, lo1, hi1, ag0, ag1);
                        dot16_e4m3(v[m], lo0, hi0, lo1, hi1, au0, au1);
                    } else {
                        const float4 lo = xlo[c], hi = xhi[c];
                        dot8_2(g[m], lo, hi, ag0, ag1);
                        dot8_2(v[m], lo, hi, au0, au1);
                    }
                }
            }
            float gs = warp_sum(ag0 + ag1), us = warp_sum(au0 + au1);
            if constexpr (F8) {   // the row scales turn the sums of q * x into g and u
                if (lane == 0) {
                    const size_t row = (size_t)s_idx[j] * 2 * I + f;
                    gs *= __ldg(a.gu_scale + row);
                    us *= __ldg(a.gu_scale + row + I);
                }
            }
            if (lane == 0) a.h[(size_t)j * I + f] = to_bf16_bits(silu(gs) * us);
        };
        auto fmod_i = [&](int x) { return x >= I ? x - I : x; };
        int ja = qj, fa = fmod_i(qf);
        bool ha = qj < k;
        if (ha) {
            advance(kDecWarps);
            load_pair(ja, fa, ga, ua);
        }
        while (ha) {
            const int jb = qj, fb = fmod_i(qf);
            const bool hb = qj < k;
            if (hb) {
                advance(kDecWarps);
                load_pair(jb, fb, gb, ub);
            }
            finish_pair(ja, fa, ga, ua);
            if (!hb) break;
            ja = qj;
            fa = fmod_i(qf);
            ha = qj < k;
            if (ha) {
                advance(kDecWarps);
                load_pair(ja, fa, ga, ua);
            }
            finish_pair(jb, fb, gb, ub);
        }
    }
    named_barrier_sync(1, kDecWarps * 32);
    if (ct == 0) grid_sync(a.bar, (unsigned)(G + a.extra_blocks), a.err, a.wait_ns);
    named_barrier_sync(1, kDecWarps * 32);
    // every block of this grid is resident (all passed the barrier): the next kernel may
    // launch and wait for SMs without starving this grid's barrier
    pdl_launch_dependents();
    // h of every slot (written by other blocks in this launch: read through L2)
    for (int q = ct; q < k * I / 8; q += kDecWarps * 32)
        reinterpret_cast<uint4*>(hs)[q] = __ldcg(reinterpret_cast<const uint4*>(a.h) + q);
    named_barrier_sync(1, kDecWarps * 32);

    // down: stage i (slot i's rows d0..d1-1) is taken by the warp that owns its ring slot,
    // (i % NS) % 8: every slot has one consumer, which takes the slot's rounds in order (a
    // wait for round r must not start before round r - 1 of the slot has completed: a parity
    // wait one phase ahead would return at once).  The rows times h_i is a small contraction
    // (16-row tiles x I x one column): warp MMAs m16n8k16 with the rows as A (ldmatrix from
    // the padded stage) and h_i as column 0 of B (lanes 0-3 hold it, the other columns are 0),
    // FP32 accumulators in four chains over K; column 0 of D is in lanes 0, 4, ..., 28.
    if constexpr (F8) {
        // E4M3 rows (packed, I bytes each) times h_i on CUDA cores: rows four at a time, lanes
        // 8g..8g+7 on row g + 4q, lane 8g + l8 the 16-byte pieces l8, l8 + 8, ... (16 values
        // each), then the row scale.  The expert of each slot is read once the selection has
        // published all k (it has long finished by now).
        {
            const uint64_t t0 = globaltimer_ns();
            while (*reinterpret_cast<volatile int*>(&s_nsel) < k)
                if (globaltimer_ns() - t0 > a.wait_ns) {
                    set_error(a.err, kErrWaitMma);
                    break;
                }
        }
        const int g = lane >> 3, l8 = lane & 7;
        const int PC = I / 16;
        bool ok = true;
        for (int s = cw; s < NS && ok; s += kDecWarps)
            for (int i = s, r = 0; i < ND; i += NS, ++r) {
                if (!mbar_wait(full + s, r & 1, a.err, kErrWaitMma, a.wait_ns)) {
                    ok = false;
                    break;
                }
                const uint4* hrow = reinterpret_cast<const uint4*>(hs + (size_t)i * I);
                const float* sc = a.dn_scale + (size_t)(*reinterpret_cast<volatile int*>(&s_idx[i])) * D + d0;
                for (int q = 0; q * 4 < nd; ++q) {
                    const int rr = q * 4 + g;
                    float acc0 = 0.f, acc1 = 0.f;
                    if (rr < nd) {
                        const uint4* wr = reinterpret_cast<const uint4*>(ring + (size_t)s * L.sb + (size_t)rr * L.rs);
                        for (int c = l8; c < PC; c += 8) dot16_e4m3_bf16(wr[c], hrow[2 * c], hrow[2 * c + 1], acc0, acc1);
                    }
                    float v = acc0 + acc1;
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    if (rr < nd && l8 == 0) val[(size_t)i * nd_max + rr] = v * __ldg(sc + rr);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + s);
            }
    } else {
        const int grp = lane >> 2, tig = lane & 3;
        const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;   // ldmatrix: this lane's row
        const int akof = (lane >> 4) * 16;                     // and its 16-byte half of the k step
        const uint32_t* h32 = reinterpret_cast<const uint32_t*>(hs);
        const int KS = I / 16;
        bool ok = true;
        for (int s = cw; s < NS && ok; s += kDecWarps)
          for (int i = s, r = 0; i < ND; i += NS, ++r) {
            if (!mbar_wait(full + s, r & 1, a.err, kErrWaitMma, a.wait_ns)) {
                ok = false;
                break;
            }
            const uint32_t* hi32 = h32 + (size_t)i * (I / 2);
            for (int mt = 0; mt * 16 < nd; ++mt) {
                const uint32_t abase = smem_u32(ring + (size_t)s * L.sb + (size_t)(mt * 16 + arow) * L.rs + akof);
                float c[4][4];
#pragma unroll
                for (int q = 0; q < 4; ++q) c[q][0] = c[q][1] = c[q][2] = c[q][3] = 0.f;
                int ks = 0;
                for (; ks + 4 <= KS; ks += 4) {
                    // the fragment loads of four k steps first, then their MMAs (the asm
                    // statements issue in program order; an MMA waits only for its own loads)
                    uint32_t af[4][4], bf[4][2];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        ldmatrix_x4(abase + (uint32_t)(ks + q) * 32u, af[q][0], af[q][1], af[q][2], af[q][3]);
                        bf[q][0] = grp == 0 ? hi32[(ks + q) * 8 + tig] : 0u;
                        bf[q][1] = grp == 0 ? hi32[(ks + q) * 8 + 4 + tig] : 0u;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        mma_bf16_16816(c[q], af[q][0], af[q][1], af[q][2], af[q][3], bf[q][0], bf[q][1]);
                }
                for (; ks < KS; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(abase + (uint32_t)ks * 32u, a0, a1, a2, a3);
                    const uint32_t b0 = grp == 0 ? hi32[ks * 8 + tig] : 0u;
                    const uint32_t b1 = grp == 0 ? hi32[ks * 8 + 4 + tig] : 0u;
                    mma_bf16_16816(c[0], a0, a1, a2, a3, b0, b1);
                }
                if (tig == 0) {
                    const int r0 = mt * 16 + grp, r1 = r0 + 8;
                    if (r0 < nd) val[(size_t)i * nd_max + r0] = (c[0][0] + c[1][0]) + (c[2][0] + c[3][0]);
                    if (r1 < nd) val[(size_t)i * nd_max + r1] = (c[0][2] + c[1][2]) + (c[2][2] + c[3][2]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);
          }
    }
    named_barrier_sync(2, kDecThreads);   // with the copy warp: s_w is written
    // combine: the k weighted expert outputs in slot order, then the residual
    for (int dd = ct; dd < nd; dd += kDecWarps * 32) {
        const int d = d0 + dd;
        float acc = 0.f;
        for (int s = 0; s < k; ++s) {
            const float pr = __fmul_rn(s_w[s], val[(size_t)s * nd_max + dd]);
            acc = s == 0 ? pr : __fadd_rn(acc, pr);
        }
        if (a.residual) {
            // out may be the residual buffer: read before the write below, past L1
            const unsigned short r = __ldcg(reinterpret_cast<const unsigned short*>(a.residual) + d);
            acc = __fadd_rn(acc, __uint_as_float((uint32_t)r << 16));
        }
        if (a.out_f32) a.out_f32[d] = acc;
        a.out[d] = to_bf16_bits(acc);
    }
}

int decode_stages(int T, int D, int E, int k, int I, int blocks, bool f8) {
    if (T != 1 || k > kMaxK || D > kDecMaxD || blocks < 1) return 0;
    if (D % 64 != 0 || I % 16 != 0 || E > 512) return 0;
    const int nd_max = (D + blocks - 1) / blocks;
    const DecodeLayout fixed = decode_layout(D, k, I, nd_max, 0, f8);
    const long long room = (long long)kDecSmemBudget - (long long)fixed.total;
    const long long per = (long long)fixed.sb + 16;   // a stage and its two barriers
    long long st = room > 0 ? room / per : 0;
    if (st > kDecMaxStages) st = kDecMaxStages;
    return st >= kDecMinStages ? (int)st : 0;
}

template <int VPL, bool F8>
static cudaError_t launch_decode_t(const DecodeArgs& a, int blocks, bool pdl, cudaStream_t s) {
    const int nd_max = (a.D + blocks - 1) / blocks;
    const size_t smem = decode_layout(a.D, a.k, a.I, nd_max, a.stages, F8).total;
    auto kern = decode_block_kernel<VPL, F8>;
    cudaError_t e = ensure_smem_attr((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, dim3(blocks), dim3(kDecThreads), smem, s, pdl, a);
}

cudaError_t launch_decode(const DecodeArgs& a, int blocks, bool pdl, cudaStream_t s) {
    if (a.stages < kDecMinStages) return cudaErrorInvalidValue;
    if (a.W_gu8) {
        if (a.E <= 128) return launch_decode_t<4, true>(a, blocks, pdl, s);
        if (a.E <= 256) return launch_decode_t<8, true>(a, blocks, pdl, s);
        return launch_decode_t<16, true>(a, blocks, pdl, s);
    }
    if (a.E <= 128) return launch_decode_t<4, false>(a, blocks, pdl, s);
    if (a.E <= 256) return launch_decode_t<8, false>(a, blocks, pdl, s);
    return launch_decode_t<16, false>(a, blocks, pdl, s);
}

}  // namespace moe
