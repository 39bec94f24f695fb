// Tensor-core (tcgen05 + TMA) kernels for the two passes of Eq. (1), "Sana:
// Efficient High-Resolution Image Synthesis with Linear Diffusion Transformers",
// section 2.1, with the per-head QK-RMSNorm of "SANA 1.5 ...", section "Model
// architecture" (QK Norm bullet).  bf16 inputs and outputs, fp32 accumulation.
//
// Both passes are HBM-bound (16.5 flop per byte); the D x (D+1) contractions go
// to the tensor cores only because CUDA-core FMAs cannot keep up with HBM here.
// Both kernels are persistent: one CTA per SM walks a contiguous, balanced range
// of a flat work list, so there is no tail wave and setup is paid once per SM.
// Small UMMAs cost about the same issue time whatever their N, so both passes
// are laid out to issue as few of them per byte as the operand shapes allow.
//
// Pass 1, kv_partials_persistent.  Work item = one 64-token stage of one row
// (b, g), g a group of 4 heads (128 channels).  Per stage one UMMA chain
//     D[(h,d), (h',e)] += sum_t phi(K)[t,(h,d)] V[t,(h',e)]       (M=128, N=128, K=64)
// whose diagonal blocks h == h' are the state's value columns.  The normaliser
// column sum_t phi(K)[t,(h,d)] is summed on the CUDA cores by the warps that
// compute phi(K) (from the same bf16-rounded values the UMMA reads).  TMA brings
// K and V tiles with the 128-byte swizzle, [token][channel]; the transform warps
// rewrite K in place as phi(K) = ReLU(g * k / rms(k)), which makes it the
// MN-major A operand; V already is the MN-major B operand.  At the end of each
// row segment the epilogue warps store the segment's partial state, transposed
// ([e][d], coalesced); a row's partials are summed in CTA order by the consumer
// (pass 2's operand builder, or the combine kernel), so results are bitwise
// reproducible and pass 1 needs no counters or atomics.
//
// Pass 2, apply_persistent.  Work item = one 128-token tile of one row (b, p), p a
// pair of heads (64 channels).  A builder warp sums the row's partial states (or
// reads a given state) and writes the B operand of both heads, K-major, one
// 128-byte row per output column n: rows 0..31 the bf16 "hi" part of the value
// columns, row 32 / 33 the hi / lo parts of the normaliser column, rows 48..79 the
// "lo" parts (x - bf16(x)) of the value columns, so the state keeps ~16 mantissa
// bits.  The workers rewrite the Q tile in place as phi(Q) (K-major A operand);
// per head two UMMAs (M=128, N=80, K=16 each) give
//     D[t, n] = sum_d phi(Q)[t,d] Bop[n, d]
// and the workers form num_e = D[e] + D[48+e], den = D[32] + D[33],
// O = num * (1 / (den + eps)), write O over the tile; a store warp TMA-stores it
// and hands the slot back to the producer as soon as the store has read it.
//
// Launch chaining (programmatic dependent launch): pass 1 waits for the previous
// grid before touching memory and only then lets pass 2 launch, so pass 2 may
// read Q and the gains early; pass 2 reads what pass 1 wrote only after its own
// wait.  Pass 2 lets the next grid launch at once; whatever follows waits for it.
//
// TMEM: warp w reads lanes 32 * (w % 4) .. + 31; D row i is lane i.
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"

namespace sana {

// x[i] = ReLU(g[i] * x[i] * r) (kScaleByRms) or ReLU(g[i] * x[i]) for one head's 32
// values, the gains read from shared memory eight at a time as 16-byte loads (g
// must be 16-byte aligned: the gain arrays start 1024-byte aligned and a head's
// gains are 128 bytes apart).
template <bool kScaleByRms>
__device__ __forceinline__ void scale_relu32(float* x, const float* g, float r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 v = reinterpret_cast<const float4*>(g)[c];
        const float gv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
            x[4 * c + u] = kScaleByRms ? fmaxf(gv[u] * (x[4 * c + u] * r), 0.f)
                                       : fmaxf(gv[u] * x[4 * c + u], 0.f);
    }
}

// The feature map on 32 values held as 4 swizzled 16-byte chunks of row `row`,
// starting at chunk `chunk0`, rewritten in place as bf16.  g points at the
// head's 32 gains in shared memory (ignored with the norm off).
//   scale_by_rms: phi = ReLU(g * x * r) with r = rsqrt(mean(x^2) + eps)
//   otherwise   : ReLU(g * x) is written and r is returned for the caller to
//                 apply later (it is a positive per-token factor).
//   norm off    : ReLU(x); returns 1.
//   zero        : writes zeros (rows past N, heads past H); returns 1.
// sum (optional): the 32 bf16-rounded results are added to sum[0..31].
template <bool kScaleByRms>
__device__ __forceinline__ float phi_inplace_sw128(uint8_t* tile, int row, int chunk0,
                                                   const float* g, float eps, bool norm,
                                                   bool zero, float* sum = nullptr) {
    uint4 u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
        u[c] = *reinterpret_cast<const uint4*>(tile + sw128_offset(row, chunk0 + c));
    float x[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        x[8 * c + 0] = bf16lo(u[c].x); x[8 * c + 1] = bf16hi(u[c].x);
        x[8 * c + 2] = bf16lo(u[c].y); x[8 * c + 3] = bf16hi(u[c].y);
        x[8 * c + 4] = bf16lo(u[c].z); x[8 * c + 5] = bf16hi(u[c].z);
        x[8 * c + 6] = bf16lo(u[c].w); x[8 * c + 7] = bf16hi(u[c].w);
    }
    float r = 1.f;
    if (norm && !zero) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;      // four chains, not one
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            s0 = fmaf(x[i], x[i], s0);
            s1 = fmaf(x[i + 1], x[i + 1], s1);
            s2 = fmaf(x[i + 2], x[i + 2], s2);
            s3 = fmaf(x[i + 3], x[i + 3], s3);
        }
        r = rsqrtf(((s0 + s1) + (s2 + s3)) * (1.f / kD) + eps);
        scale_relu32<kScaleByRms>(x, g, r);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = zero ? 0.f : fmaxf(x[i], 0.f);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4*>(tile + sw128_offset(row, chunk0 + c)) = w;
        if (sum) {
            sum[8 * c + 0] += bf16lo(w.x); sum[8 * c + 1] += bf16hi(w.x);
            sum[8 * c + 2] += bf16lo(w.y); sum[8 * c + 3] += bf16hi(w.y);
            sum[8 * c + 4] += bf16lo(w.z); sum[8 * c + 5] += bf16hi(w.z);
            sum[8 * c + 6] += bf16lo(w.w); sum[8 * c + 7] += bf16hi(w.w);
        }
    }
    return kScaleByRms ? 1.f : r;
}

// Two items of phi_inplace_sw128 at once: both items' loads are issued before
// either item's stores, so their latencies overlap (the compiler cannot reorder
// shared-memory stores and loads that may alias).
template <bool kScaleByRms>
__device__ __forceinline__ void phi2_inplace_sw128(uint8_t* const tile[2], const int row[2],
                                                   const int chunk0[2], const float* const g[2],
                                                   float eps, bool norm, const bool zero[2],
                                                   float r_out[2], float* sum,
                                                   const float* wsum = nullptr) {
    uint4 u[2][4];
#pragma unroll
    for (int it = 0; it < 2; ++it)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            u[it][c] = *reinterpret_cast<const uint4*>(tile[it] + sw128_offset(row[it], chunk0[it] + c));
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        float x[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            x[8 * c + 0] = bf16lo(u[it][c].x); x[8 * c + 1] = bf16hi(u[it][c].x);
            x[8 * c + 2] = bf16lo(u[it][c].y); x[8 * c + 3] = bf16hi(u[it][c].y);
            x[8 * c + 4] = bf16lo(u[it][c].z); x[8 * c + 5] = bf16hi(u[it][c].z);
            x[8 * c + 6] = bf16lo(u[it][c].w); x[8 * c + 7] = bf16hi(u[it][c].w);
        }
        float r = 1.f;
        if (norm && !zero[it]) {
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                s0 = fmaf(x[i], x[i], s0);
                s1 = fmaf(x[i + 1], x[i + 1], s1);
                s2 = fmaf(x[i + 2], x[i + 2], s2);
                s3 = fmaf(x[i + 3], x[i + 3], s3);
            }
            r = rsqrtf(((s0 + s1) + (s2 + s3)) * (1.f / kD) + eps);
            scale_relu32<kScaleByRms>(x, g[it], r);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = zero[it] ? 0.f : fmaxf(x[i], 0.f);
        }
        r_out[it] = kScaleByRms ? 1.f : r;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            u[it][c].x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
            u[it][c].y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
            u[it][c].z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
            u[it][c].w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
            if (sum && wsum) {                      // column sums weighted per item
                const float wv = wsum[it];
                sum[8 * c + 0] = fmaf(bf16lo(u[it][c].x), wv, sum[8 * c + 0]);
                sum[8 * c + 1] = fmaf(bf16hi(u[it][c].x), wv, sum[8 * c + 1]);
                sum[8 * c + 2] = fmaf(bf16lo(u[it][c].y), wv, sum[8 * c + 2]);
                sum[8 * c + 3] = fmaf(bf16hi(u[it][c].y), wv, sum[8 * c + 3]);
                sum[8 * c + 4] = fmaf(bf16lo(u[it][c].z), wv, sum[8 * c + 4]);
                sum[8 * c + 5] = fmaf(bf16hi(u[it][c].z), wv, sum[8 * c + 5]);
                sum[8 * c + 6] = fmaf(bf16lo(u[it][c].w), wv, sum[8 * c + 6]);
                sum[8 * c + 7] = fmaf(bf16hi(u[it][c].w), wv, sum[8 * c + 7]);
            } else if (sum) {
                sum[8 * c + 0] += bf16lo(u[it][c].x); sum[8 * c + 1] += bf16hi(u[it][c].x);
                sum[8 * c + 2] += bf16lo(u[it][c].y); sum[8 * c + 3] += bf16hi(u[it][c].y);
                sum[8 * c + 4] += bf16lo(u[it][c].z); sum[8 * c + 5] += bf16hi(u[it][c].z);
                sum[8 * c + 6] += bf16lo(u[it][c].w); sum[8 * c + 7] += bf16hi(u[it][c].w);
            }
        }
    }
#pragma unroll
    for (int it = 0; it < 2; ++it)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(tile[it] + sw128_offset(row[it], chunk0[it] + c)) = u[it][c];
}

// Copy n <= kMax floats (a gain vector) from global to shared memory as thread
// `tid` of kThreadsT: each thread issues up to kBatch of its loads before any
// store, so the copy costs ceil(kMax / (kThreadsT kBatch)) memory round trips
// instead of one per strided loop iteration.
template <int kMax, int kThreadsT, int kBatch = 8>
__device__ __forceinline__ void load_gains(float* dst, const float* __restrict__ src, int n,
                                           int tid) {
    constexpr int kPer = (kMax + kThreadsT - 1) / kThreadsT;
#pragma unroll 1
    for (int u0 = 0; u0 < kPer; u0 += kBatch) {
        if (tid + u0 * kThreadsT >= n) break;
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = tid + (u0 + u) * kThreadsT;
            v[u] = (u0 + u < kPer && i < n) ? __ldg(src + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = tid + (u0 + u) * kThreadsT;
            if (u0 + u < kPer && i < n) dst[i] = v[u];
        }
    }
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
    return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// Sum of 32 per-lane values over the 32 lanes of a warp (butterfly
// reduce-scatter): on return lane l holds the total of entry l in v[0].  The
// order of the additions is fixed, so the result is reproducible.
__device__ __forceinline__ void warp_reduce_scatter32(float* v, int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
}

// ============================================================================ pass 1
namespace p1 {
constexpr int kGroupHeads = 4;                     // heads per row (UMMA M = 128)
constexpr int kStageTok = 64;                      // tokens per stage
constexpr int kBoxBytes = kStageTok * 128;         // kStageTok tokens x 64 channels
constexpr int kStageBytes = 4 * kBoxBytes;         // [K box 0 | K box 1 | V box 0 | V box 1]
constexpr int kRingBytes = 192 * 1024;
constexpr int kStages = kRingBytes / kStageBytes;  // 6
constexpr int kAccCols = 128;                      // one accumulator (4 heads x 32 columns)
constexpr int kTmemCols = 2 * kAccCols;            // double-buffered across row segments
constexpr int kTransformWarps = 8;                 // two groups of 4, alternating stages
constexpr int kEpilogueWarps = 4;
constexpr int kThreads = 32 * (2 + kTransformWarps + kEpilogueWarps);
constexpr int kGainCache = 4096;                   // channels whose gains live in smem
constexpr int kKsumFloats = kTransformWarps * 32;  // each transform warp's 32 column sums
constexpr int kSmemBytes = 1024 + kRingBytes + kGainCache * 4 + 2 * kKsumFloats * 4 + 512;
// Warp w of a transform group handles head w of the row, thread l of the warp
// token rows l and l + 32, in every stage of its group.
static_assert(kStageTok == 64 && kGroupHeads == 4, "two items per transform thread");
// The two transform groups take alternate stages; with an even slot count every
// slot belongs to one group, so each mbarrier phase is awaited in order (an odd
// count would let a group test a slot's next phase before the current one
// completed).
static_assert(kStages >= 2 && kStages % 2 == 0, "ring slots must be even");
}  // namespace p1

struct P1Args {
    const float* gk;     // gains [C], or nullptr with the norm off
    const float* w;      // kWeighted: per token-head weights [B][H][N] of the normaliser
                         // column (sum_t phi(K)[t] w[t] in place of sum_t phi(K)[t])
    float* part;         // partial states [B][H][Smax][D+1][D]  (column e major);
                         // chunked: [B][H][Cc][Smax][D+1][D]
    int64_t T;           // work items: B * G rows x R stages (chunked: B * G * Cc rows)
    int N, H, G, R, Smax, P;
    float eps;
    int norm;
    int Cc;              // chunked: chunks of R stages each (b, g) sequence is cut into
};

// One row per (b, g) over the whole sequence (the forward's state), or, with
// kChunked, one row per (b, g, chunk of R stages): the states of the sequence's
// chunks, which the prefix (causal) form scans.  kWeighted (the backward's
// [dS | dz] = sum_t phi(Q)_t^T [dnum_t | dden_t]): the normaliser column is
// sum_t phi(K)[t] w[t] with w per token and head.
template <bool kChunked, bool kWeighted = false>
__global__ void __launch_bounds__(p1::kThreads, 1)
kv_partials_persistent(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const P1Args a)
{
    using namespace p1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    float* sgain = (float*)(stages + kRingBytes);
    float* ksbuf = sgain + kGainCache;                  // [2][kTransformWarps][64]
    uint64_t* full = (uint64_t*)(ksbuf + 2 * kKsumFloats);
    uint64_t* aready = full + kStages;
    uint64_t* empty = aready + kStages;
    uint64_t* accfull = empty + kStages;
    uint64_t* accempty = accfull + 2;
    uint64_t* ksfull = accempty + 2;
    uint64_t* ksempty = ksfull + 2;
    uint64_t* drain = ksempty + 2;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int64_t c = blockIdx.x;
    const int64_t i0 = range_begin(c, a.T, a.P), i1 = range_begin(c + 1, a.T, a.P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.H * kD;                      // at most kGainCache (checked on the host)

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], 32 * kTransformWarps / 2);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 32 * kEpilogueWarps);
            mbar_init(&ksfull[i], 32 * kTransformWarps);
            mbar_init(&ksempty[i], 32 * kEpilogueWarps);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Nothing above touched global memory.  Wait for the previous grid, then let
    // the apply pass launch: it may read Q and its gains before its own wait.
    pdl_wait_primary();
    pdl_launch_dependents();
    bool ok = i1 > i0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; i0 + li < i1; ++li) {
                const int st = (int)(li % kStages);
                if (li >= kStages) ok = mbar_wait(&empty[st], (uint32_t)((li / kStages) - 1) & 1, 301);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R);
                const int64_t rg = kChunked ? r / a.Cc : r;                   // (b, g)
                const int b = (int)(rg / a.G), g = (int)(rg % a.G);
                const int t0 = kChunked ? (int)(r % a.Cc) * a.R : 0;         // first stage
                uint8_t* sb = stages + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                const int x = g * 128, y = (t0 + t) * kStageTok;
                tma_load_3d(sb, &tmap_k, &full[st], x, y, b);
                tma_load_3d(sb + kBoxBytes, &tmap_k, &full[st], x + 64, y, b);
                tma_load_3d(sb + 2 * kBoxBytes, &tmap_v, &full[st], x, y, b);
                tma_load_3d(sb + 3 * kBoxBytes, &tmap_v, &full[st], x + 64, y, b);
                last = li;
            }
            if (!ok) {   // let every issued copy land before the CTA can exit
                for (int st = 0; st < kStages; ++st) {
                    const int64_t li = last - ((last - st) % kStages + kStages) % kStages;
                    if (last >= 0 && li >= 0)
                        mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 302);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (whole warp,
        // one elected lane issues)
        // Ring position, phase bit and descriptors advance as counters (no divisions or
        // descriptor packing per stage).
        if (ok) {
            const uint32_t idesc = make_idesc_bf16(128, 128, true, true);
            const uint64_t k0 = make_smem_desc(smem_u32(stages), kBoxBytes, 1024, kSwizzle128B);
            const uint64_t v0 = k0 + (uint64_t)((2 * kBoxBytes) >> 4);
            const int64_t n = i1 - i0;
            int st = 0, seg = 0;
            uint32_t fpar = 0;
            int64_t t = i0 % a.R;
            for (int64_t li = 0; li < n; ++li) {
                const bool first = (li == 0) || (t == 0);
                const bool lastst = (li + 1 == n) || (t == a.R - 1);
                const int abuf = seg & 1;
                if (lane == 0) {
                    if (first && seg >= 2)
                        ok = mbar_wait(&accempty[abuf], (uint32_t)((seg >> 1) - 1) & 1, 303);
                    if (ok) ok = mbar_wait(&aready[st], fpar, 304);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + abuf * kAccCols;
                const uint64_t so = (uint64_t)((st * kStageBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kStageTok / 16; ++kk)   // 16 token rows = 2048 bytes a step
                    umma_bf16_elect(d, k0 + so + kk * 128, v0 + so + kk * 128, idesc,
                                    !(first && kk == 0));
                umma_commit_elect(&empty[st]);
                if (lastst) {
                    umma_commit_elect(&accfull[abuf]);
                    ++seg;
                }
                if (++st == kStages) { st = 0; fpar ^= 1; }
                if (++t == a.R) t = 0;
            }
            umma_commit_elect(drain);
            if (lane == 0) mbar_wait(drain, 0, 305);
            __syncwarp();
        }
    } else if (warp < 2 + kTransformWarps) {
        // ------------------------------------------------ phi(K) in place + column sums
        // Two groups of 4 warps take alternate stages, so two stages are in the
        // transform at once.  Within a stage, warp hl of a group takes head hl and
        // lane l token rows l and l + 32, so each quarter warp touches 8
        // consecutive swizzled rows; the warp's column sums are one head's.
        const int wt = threadIdx.x - 64;                 // 0..255
        const int wi = wt >> 5;                          // transform warp 0..7
        const int grp = wt >> 7;                         // stages with li % 2 == grp
        const int hl = wi & 3;                           // head within the row
        if (a.norm) load_gains<kGainCache, 32 * kTransformWarps>(sgain, a.gk, C, wt);
        named_barrier_sync(2, 32 * kTransformWarps);
        int seg = 0;
        for (int64_t sb = i0; sb < i1 && ok; ++seg) {
            // one row segment [sb, se): this group's stages are those with li % 2 == grp
            const int64_t r = sb / a.R;
            const int64_t se = (r + 1) * a.R < i1 ? (r + 1) * a.R : i1;
            const int g = (int)((kChunked ? r / a.Cc : r) % a.G);
            const int tbase = kChunked ? (int)(r % a.Cc) * a.R * kStageTok : 0;
            const int h = g * kGroupHeads + hl;
            float ks[kD];
#pragma unroll
            for (int e = 0; e < kD; ++e) ks[e] = 0.f;
            int64_t li = sb - i0;
            if ((li & 1) != grp) ++li;
            for (; i0 + li < se && ok; li += 2) {
                const int st = (int)(li % kStages);
                ok = mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 306);
                if (!ok) break;
                const int t = (int)((i0 + li) % a.R);
                uint8_t* const tl[2] = {stages + st * kStageBytes + (hl >> 1) * kBoxBytes,
                                        stages + st * kStageBytes + (hl >> 1) * kBoxBytes};
                const int rows[2] = {lane, lane + 32}, ch[2] = {(hl & 1) * 4, (hl & 1) * 4};
                const bool dead[2] = {!((tbase + t * kStageTok + lane < a.N) && (h < a.H)),
                                      !((tbase + t * kStageTok + lane + 32 < a.N) && (h < a.H))};
                const float* gg[2] = {sgain + (h < a.H ? h : 0) * kD, sgain + (h < a.H ? h : 0) * kD};
                float rr[2];
                float wv[2] = {1.f, 1.f};
                if (kWeighted) {
                    const int64_t bb = (kChunked ? r / a.Cc : r) / a.G;
                    for (int it = 0; it < 2; ++it) {
                        const int64_t tok = tbase + (int64_t)t * kStageTok + rows[it];
                        wv[it] = dead[it] ? 0.f : __ldg(a.w + (bb * a.H + h) * a.N + tok);
                    }
                }
                phi2_inplace_sw128<true>(tl, rows, ch, gg, a.eps, a.norm != 0, dead, rr, ks,
                                         kWeighted ? wv : nullptr);
                fence_proxy_async_smem();
                mbar_arrive(&aready[st]);
            }
            if (!ok) break;
            // the warp's 32 column sums (head hl, channel = lane) -> shared memory
            warp_reduce_scatter32(ks, lane);
            const int buf = seg & 1;
            if (seg >= 2) ok = mbar_wait(&ksempty[buf], (uint32_t)((seg >> 1) - 1) & 1, 308);
            if (!ok) break;
            ksbuf[buf * kKsumFloats + wi * 32 + lane] = ks[0];
            mbar_arrive(&ksfull[buf]);
            sb = se;
        }
    } else {
        // ------------------------------------------------ segment epilogue
        const int q = warp & 3;                                     // head within the row
        int seg = 0;
        for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
            const int64_t i = i0 + li;
            const int t = (int)(i % a.R);
            if (!((i + 1 == i1) || (t == a.R - 1))) continue;      // not a segment end
            const int abuf = seg & 1;
            ok = mbar_wait(&accfull[abuf], (uint32_t)(seg >> 1) & 1, 307);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + abuf * kAccCols;
            float v[kD];
            tmem_ld16(ta + 32 * q, v);
            tmem_ld16(ta + 32 * q + 16, v + 16);
            tmem_wait_ld();
            tc_fence_before_sync();
            mbar_arrive(&accempty[abuf]);
            ok = mbar_wait(&ksfull[abuf], (uint32_t)(seg >> 1) & 1, 309);
            if (!ok) break;
            // head q's column sums from transform warp q of each group, in group order
            const float* kb = ksbuf + abuf * kKsumFloats + q * 32 + lane;
            const float ks = kb[0] + kb[4 * 32];
            mbar_arrive(&ksempty[abuf]);
            ++seg;

            const int64_t r = i / a.R;
            const int64_t rg = kChunked ? r / a.Cc : r;
            const int b = (int)(rg / a.G), g = (int)(rg % a.G);
            const int slot = (int)(c - owner_cta(r * a.R, a.T, a.P));
            const int h = g * kGroupHeads + q;
            if (h < a.H) {
                // lane = d; element (e, d) at e * 32 + d: one 128-byte row per store
                const size_t bh = (size_t)b * a.H + h;
                const size_t row = kChunked ? bh * a.Cc + (size_t)(r % a.Cc) : bh;
                float* o = a.part + (row * a.Smax + slot) * kStateFloats + lane;
#pragma unroll
                for (int e = 0; e < kD; ++e) o[e * kD] = v[e];
                o[kD * kD] = ks;
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The number of partial slots of pass-1 row r (CTAs whose ranges meet it).
__host__ __device__ __forceinline__ int p1_row_slots(int64_t r, int64_t R, int64_t T, int64_t P) {
    return (int)(owner_cta(r * R + R - 1, T, P) - owner_cta(r * R, T, P) + 1);
}

// State of each (b, h) from pass-1 partials, summed in slot order: grid B * H,
// kv[d][e] = sum_s part[s][e][d].  Launched right behind pass 1.
__global__ void __launch_bounds__(256)
kv_combine_partials(const float* __restrict__ part, float* __restrict__ kv, int H, int G,
                    int64_t R, int64_t T, int64_t P, int Smax)
{
    pdl_wait_primary();
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / H, h = bh % H;
    const int ns = p1_row_slots(b * G + h / p1::kGroupHeads, R, T, P);
    const float* src = part + bh * Smax * (int64_t)kStateFloats;
    for (int idx = threadIdx.x; idx < kStateFloats; idx += blockDim.x) {
        float acc = 0.f;
        for (int s = 0; s < ns; ++s) acc += src[(int64_t)s * kStateFloats + idx];
        const int e = idx / kD, d = idx % kD;
        kv[bh * kStateFloats + d * kDP + e] = acc;
    }
}

// ============================================================================ pass 2
namespace p2 {
constexpr int kTileTok = 128;                      // UMMA M
constexpr int kPairHeads = 2;                      // 64 channels = one swizzled row
constexpr int kTileBytes = kTileTok * 128;         // 16 KB
constexpr int kStages = 10;
constexpr int kStoresInFlight = 2;                 // TMA stores the store warp keeps open
constexpr int kN = 80;                             // B rows per head (see the file comment)
constexpr int kLoRow = 48;                         // first row of the value columns' lo parts
constexpr int kDenHi = 32, kDenLo = 33;            // rows of the normaliser's hi / lo parts
static_assert(kDenHi == kD, "the normaliser column sits in B row e = D");
constexpr int kBopBytes = kN * 128;                // both heads side by side in each row
constexpr int kBopRing = 2;
constexpr int kBufCols = kPairHeads * kN;          // 160 TMEM columns per tile
constexpr int kTmemBufs = 3;
constexpr int kTmemCols = 512;
constexpr int kSlotsPerRound = 3;                  // partial slots staged per bulk copy round
constexpr int kStagingBytes = kPairHeads * kSlotsPerRound * kStateFloats * 4;
constexpr int kWorkerWarps = 16;                   // two tile groups of 8, alternating tiles
constexpr int kGroupThreads = 32 * kWorkerWarps / 2;   // a tile group: 4 quadrants x 2 heads
constexpr int kThreads = 32 * (4 + kWorkerWarps);  // TMA, UMMA, builder, store, workers
constexpr int kGainCache = 4096;
constexpr int kSmemBytes = 1024 + kStages * kTileBytes + kBopRing * kBopBytes + kStagingBytes +
                           kGainCache * 4 + 512;
static_assert(kStages % 2 == 0, "each ring slot must belong to one worker group");
static_assert(kTmemBufs * kBufCols <= kTmemCols, "TMEM buffers");
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace p2

struct P2Args {
    const float* kv;     // states [B][H][D][D+1]; nullptr: sum pass-1 partials instead
    const float* part;   // pass-1 partials [B][H][Smax1][D+1][D] (when kv is nullptr)
    const float* gq;     // gains [C] or nullptr
    int64_t T;           // work items: B * Pp rows x R tiles
    int N, H, Pp, R, P;
    int64_t T1, P1;      // pass-1 plan: items, CTAs, stages per row, groups, slots per row
    int R1, G1, Smax1;
    float eps;
    int norm;
};

__global__ void __launch_bounds__(p2::kThreads, 1)   // 640 threads: at most 96 registers
apply_persistent(const __grid_constant__ CUtensorMap tmap_q,
                 const __grid_constant__ CUtensorMap tmap_o, const P2Args a)
{
    using namespace p2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* bop = stages + kStages * kTileBytes;
    float* staging = (float*)(bop + kBopRing * kBopBytes);
    float* sgain = staging + kStagingBytes / 4;
    uint64_t* full = (uint64_t*)(sgain + kGainCache);
    uint64_t* aready = full + kStages;
    uint64_t* mmadone = aready + kStages;
    uint64_t* tready = mmadone + kStages;
    uint64_t* empty = tready + kStages;
    uint64_t* tfree = empty + kStages;
    uint64_t* bfull = tfree + kTmemBufs;
    uint64_t* bempty = bfull + kBopRing;
    uint64_t* drain = bempty + kBopRing;
    uint64_t* sready = drain + 1;
    uint64_t* bfirst = sready + 1;                // the first segment's B, built by the workers
    uint32_t* tmem_slot = (uint32_t*)(bfirst + 1);

    // The next grid may launch now; it waits for this one before touching memory.
    pdl_launch_dependents();
    const int64_t c = blockIdx.x;
    const int64_t i0 = range_begin(c, a.T, a.P), i1 = range_begin(c + 1, a.T, a.P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.H * kD;                      // at most kGainCache (checked on the host)

    if (threadIdx.x == 0) {
        mbar_init(sready, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], kGroupThreads);
            mbar_init(&mmadone[i], 1);
            mbar_init(&tready[i], kGroupThreads);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < kTmemBufs; ++i) mbar_init(&tfree[i], kGroupThreads);
        for (int i = 0; i < kBopRing; ++i) {
            mbar_init(&bfull[i], 32);
            mbar_init(&bempty[i], 1);
        }
        mbar_init(drain, 1);
        mbar_init(bfirst, kWorkerWarps * 32);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_o);
    }
    // B operand rows that never carry data stay zero
    for (int i = threadIdx.x; i < kBopRing * (kLoRow - kDenLo - 1) * 8; i += blockDim.x) {
        const int rb = i / ((kLoRow - kDenLo - 1) * 8), rem = i % ((kLoRow - kDenLo - 1) * 8);
        *reinterpret_cast<uint4*>(bop + rb * kBopBytes + (kDenLo + 1 + rem / 8) * 128 +
                                  (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    if (a.norm) load_gains<kGainCache, kThreads>(sgain, a.gq, C, threadIdx.x);
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = i1 > i0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (Q tiles)
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; i0 + li < i1; ++li) {
                const int st = (int)(li % kStages);
                if (li >= kStages) ok = mbar_wait(&empty[st], (uint32_t)((li / kStages) - 1) & 1, 401);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                mbar_arrive_expect_tx(&full[st], kTileBytes);
                tma_load_3d(stages + st * kTileBytes, &tmap_q, &full[st], p * 64, t * kTileTok, b);
                last = li;
            }
            if (!ok) {
                for (int st = 0; st < kStages; ++st) {
                    const int64_t li = last - ((last - st) % kStages + kStages) % kStages;
                    if (last >= 0 && li >= 0)
                        mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 402);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (whole warp,
        // one elected lane issues)
        // Ring / TMEM positions and phase bits advance as counters, and descriptors are
        // stepped from precomputed ones (their start address is in 16-byte units).
        if (ok) {
            const uint32_t idesc = make_idesc_bf16(128, kN, false, false);
            const uint64_t a0 = make_smem_desc(smem_u32(stages), 16, 1024, kSwizzle128B);
            const uint64_t b0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
            const int64_t n = i1 - i0;
            int st = 0, tb = 0, seg = 0;
            uint32_t fpar = 0, tpar = 0;
            int64_t t = i0 % a.R;
            for (int64_t li = 0; li < n; ++li) {
                const bool first = (li == 0) || (t == 0);
                const bool lastt = (li + 1 == n) || (t == a.R - 1);
                const int rb = seg & 1;
                if (lane == 0) {
                    if (first)
                        ok = seg == 0 ? mbar_wait(bfirst, 0, 403)
                                      : mbar_wait(&bfull[rb], (uint32_t)((seg - 1) >> 1) & 1, 403);
                    if (ok) ok = mbar_wait(&aready[st], fpar, 404);
                    if (ok && li >= kTmemBufs) ok = mbar_wait(&tfree[tb], tpar ^ 1, 405);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t ad = a0 + (uint64_t)((st * kTileBytes) >> 4);
                const uint64_t bd = b0 + (uint64_t)((rb * kBopBytes) >> 4);
                const uint32_t d = tmem + tb * kBufCols;
                umma_bf16_elect(d, ad, bd, idesc, false);
                umma_bf16_elect(d, ad + 2, bd + 2, idesc, true);
                umma_bf16_elect(d + kN, ad + 4, bd + 4, idesc, false);
                umma_bf16_elect(d + kN, ad + 6, bd + 6, idesc, true);
                umma_commit_elect(&mmadone[st]);
                if (lastt) {
                    umma_commit_elect(&bempty[rb]);
                    ++seg;
                }
                if (++st == kStages) { st = 0; fpar ^= 1; }
                if (++tb == kTmemBufs) { tb = 0; tpar ^= 1; }
                if (++t == a.R) t = 0;
            }
            umma_commit_elect(drain);
            if (lane == 0) mbar_wait(drain, 0, 406);
            __syncwarp();
        }
    } else if (warp == 2) {
        // ------------------------------------------------ B operand builder
        // Every row segment after the first (the workers build the first one): the
        // pair's state S_j[d][e] (j = head of the pair) lands in
        // registers, lane = d: either the sum of the pass-1 partials of the row, slot
        // by slot in slot order (bulk copies of up to kSlotsPerRound slots at a time),
        // or the given state.  Lane pairs (d, d + 1) then write one bf16x2 each: even
        // lanes the hi parts, odd lanes the lo parts.
        int seg = 0;
        uint32_t sphase = 0;
        for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
            const int64_t i = i0 + li;
            if (!(li == 0 || i % a.R == 0)) continue;              // not a segment start
            const int rb = seg & 1;
            if (seg == 0) {
                ++seg;
                continue;
            }
            if (seg >= 2) ok = mbar_wait(&bempty[rb], (uint32_t)((seg >> 1) - 1) & 1, 407);
            if (!ok) break;
            if (seg == 1) pdl_wait_primary();                     // the states come from pass 1
            const int64_t r = i / a.R;
            const int b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h0 = p * kPairHeads;
            const int nh = min(kPairHeads, a.H - h0);
            uint8_t* dst = bop + rb * kBopBytes;
            const int d0 = lane & ~1;                              // even d of the lane pair
            int ns = 1;
            if (a.kv == nullptr)
                ns = p1_row_slots((int64_t)b * a.G1 + h0 / p1::kGroupHeads, a.R1, a.T1, a.P1);
            // heads one at a time (registers); the bulk copies of a round bring both
            for (int j = 0; j < kPairHeads && ok; ++j) {
                float acc[kDP];
#pragma unroll
                for (int e = 0; e < kDP; ++e) acc[e] = 0.f;
                for (int s0 = 0; s0 < ns && ok; s0 += kSlotsPerRound) {
                    const int n = min(kSlotsPerRound, ns - s0);
                    if (j == 0 || ns > kSlotsPerRound) {          // (re)fill the staging area
                        __syncwarp();
                        if (lane == 0) {
                            if (a.kv == nullptr) {
                                mbar_arrive_expect_tx(sready, (uint32_t)(nh * n * kStateFloats * 4));
                                for (int jj = 0; jj < nh; ++jj)
                                    bulk_load(staging + jj * kSlotsPerRound * kStateFloats,
                                              a.part + (((size_t)b * a.H + h0 + jj) * a.Smax1 + s0) *
                                                           kStateFloats,
                                              (uint32_t)(n * kStateFloats * 4), sready);
                            } else {
                                mbar_arrive_expect_tx(sready, (uint32_t)(nh * kStateFloats * 4));
                                bulk_load(staging, a.kv + ((size_t)b * a.H + h0) * kStateFloats,
                                          (uint32_t)(nh * kStateFloats * 4), sready);
                            }
                        }
                        ok = mbar_wait(sready, sphase, 410);
                        sphase ^= 1;
                        if (!ok) break;
                    }
                    if (j >= nh) continue;                        // missing head: zeros
                    if (a.kv == nullptr) {
                        for (int s = 0; s < n; ++s)
#pragma unroll
                            for (int e = 0; e < kDP; ++e)
                                acc[e] += staging[(j * kSlotsPerRound + s) * kStateFloats + e * kD + lane];
                    } else {
#pragma unroll
                        for (int e = 0; e < kDP; ++e) acc[e] = staging[j * kStateFloats + lane * kDP + e];
                    }
                }
                if (!ok) break;
                const int chunk = j * 4 + d0 / 8, off = (d0 % 8) * 2;
#pragma unroll
                for (int e = 0; e < kDP; ++e) {
                    const float x = acc[e];
                    const float xp = __shfl_xor_sync(0xffffffffu, x, 1);
                    const float xe = (lane & 1) ? xp : x, xo = (lane & 1) ? x : xp;
                    const float he = __bfloat162float(__float2bfloat16_rn(xe));
                    const float ho = __bfloat162float(__float2bfloat16_rn(xo));
                    const int row = (lane & 1) ? (e < kD ? kLoRow + e : kDenLo) : e;
                    const uint32_t w = (lane & 1) ? pack_bf16x2(xe - he, xo - ho) : pack_bf16x2(he, ho);
                    *reinterpret_cast<uint32_t*>(dst + sw128_offset(row, chunk) + off) = w;
                }
            }
            if (!ok) break;
            fence_proxy_async_smem();
            __syncwarp();
            mbar_arrive(&bfull[rb]);
            ++seg;
        }
    } else if (warp == 3) {
        // ------------------------------------------------ output stores
        // Tiles go out in order; a slot returns to the producer as soon as its
        // store has read it.
        if (lane == 0 && ok) {
            int64_t li = 0;
            for (; i0 + li < i1 && ok; ++li) {
                const int st = (int)(li % kStages);
                ok = mbar_wait(&tready[st], (uint32_t)(li / kStages) & 1, 412);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                tma_store_3d(&tmap_o, stages + st * kTileBytes, p * 64, t * kTileTok, b);
                bulk_commit_group();
                if (li >= kStoresInFlight - 1) {       // the oldest store in flight has read its tile
                    bulk_wait_group_read<kStoresInFlight - 1>();
                    mbar_arrive(&empty[(li - (kStoresInFlight - 1)) % kStages]);
                }
            }
            bulk_wait_group_read<0>();
            for (int64_t lj = li - (kStoresInFlight - 1) > 0 ? li - (kStoresInFlight - 1) : 0; lj < li; ++lj)
                mbar_arrive(&empty[lj % kStages]);
            bulk_wait_group<0>();
        }
    } else {
        // ------------------------------------------------ phi(Q), epilogue
        // Two tile groups of 8 warps take alternate tiles; in a group, warp w takes
        // TMEM quadrant w % 4 (token rows 32 (w % 4) ..) and head (w / 4) % 2 of the pair.
        const int wi = warp - 4;                          // 0..15
        const int grp = wi >> 3;                          // tiles with li % 2 == grp
        const int j = (wi >> 2) & 1;                      // head of the pair
        const int q = warp & 3;                           // TMEM lane quadrant
        const int row = 32 * q + lane;                    // token row of the tile

        // The per-token factor r = rsqrt(mean(q^2) + eps) of phi(Q) is positive, so it
        // is left out of the A operand and applied in the epilogue:
        //   O = (r num') / (r den' + eps),  num', den' computed with ReLU(g * q).
        auto transform = [&](int64_t li, float& rq) -> bool {
            const int st = (int)(li % kStages);
            if (!mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 408)) return false;
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), p = (int)(r % a.Pp);
            const int h = p * kPairHeads + j;
            const bool live = (t * kTileTok + row < a.N) && h < a.H;
            rq = phi_inplace_sw128<false>(stages + st * kTileBytes, row, j * 4,
                                          sgain + (live ? h : 0) * kD, a.eps, a.norm != 0, !live);
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
            return true;
        };
        auto epilogue = [&](int64_t li, float rq) -> bool {
            const int st = (int)(li % kStages), tb = (int)(li % kTmemBufs);
            if (!mbar_wait(&mmadone[st], (uint32_t)(li / kStages) & 1, 409)) return false;
            tc_fence_after_sync();
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * kBufCols + j * kN;
            float hi[kD + 2], lo[kD];
            tmem_ld16(ta, hi);
            tmem_ld16(ta + 16, hi + 16);
            tmem_ld2(ta + kDenHi, hi + kD);
            tmem_ld16(ta + kLoRow, lo);
            tmem_ld16(ta + kLoRow + 16, lo + 16);
            tmem_wait_ld();
            tc_fence_before_sync();
            mbar_arrive(&tfree[tb]);
            const float den = hi[kD] + hi[kD + 1];
            const float scale = rq * __frcp_rn(fmaf(rq, den, a.eps));
            uint8_t* tile = stages + st * kTileBytes;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float o[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) o[u] = (hi[8 * cc + u] + lo[8 * cc + u]) * scale;
                uint4 w;
                w.x = pack_bf16x2(o[0], o[1]);
                w.y = pack_bf16x2(o[2], o[3]);
                w.z = pack_bf16x2(o[4], o[5]);
                w.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4*>(tile + sw128_offset(row, j * 4 + cc)) = w;
            }
            fence_proxy_async_smem();
            mbar_arrive(&tready[st]);
            return true;
        };

        // The first segment's B operand, built by all worker threads at once with plain
        // loads: one round trip to memory instead of the builder's rounds of bulk
        // copies, which would otherwise stand between pass 1's end and the first UMMA.
        // Thread item (j, e, dp): S_j[e][2dp], S_j[e][2dp + 1], consecutive threads
        // along d (coalesced in the partials' [e][d] layout); a thread's items and up
        // to kBatch slots of each are loaded before any is summed.  Slots are summed
        // in the builder's order, so the state is the same bit for bit.
        auto build_first = [&]() {
            constexpr int kItems = kPairHeads * kDP * (kD / 2);
            constexpr int kWorkers = kWorkerWarps * 32;
            constexpr int kPer = (kItems + kWorkers - 1) / kWorkers;
            constexpr int kBatch = 8;
            pdl_wait_primary();                                  // the states come from pass 1
            const int64_t r = i0 / a.R;
            const int b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int h0 = p * kPairHeads, nh = min(kPairHeads, a.H - h0);
            const int ns = a.kv == nullptr
                               ? p1_row_slots((int64_t)b * a.G1 + h0 / p1::kGroupHeads, a.R1, a.T1, a.P1)
                               : 1;
            const int tid = threadIdx.x - 128;
            float x0[kPer], x1[kPer];
            size_t off[kPer];
            bool live[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int it = tid + u * kWorkers;
                const int dp = it % (kD / 2), e = (it / (kD / 2)) % kDP, jj = it / (kD / 2 * kDP);
                live[u] = it < kItems && jj < nh;
                const size_t bh = (size_t)b * a.H + h0 + jj;
                off[u] = a.kv == nullptr ? bh * a.Smax1 * kStateFloats + e * kD + 2 * dp
                                         : bh * kStateFloats + 2 * dp * kDP + e;
                x0[u] = 0.f;
                x1[u] = 0.f;
            }
            if (a.kv == nullptr) {
                for (int s0 = 0; s0 < ns; s0 += kBatch) {
                    float2 v[kBatch][kPer];
#pragma unroll
                    for (int ss = 0; ss < kBatch; ++ss)
#pragma unroll
                        for (int u = 0; u < kPer; ++u)
                            v[ss][u] = live[u] && s0 + ss < ns
                                           ? __ldcg(reinterpret_cast<const float2*>(
                                                 a.part + off[u] + (size_t)(s0 + ss) * kStateFloats))
                                           : make_float2(0.f, 0.f);
#pragma unroll
                    for (int ss = 0; ss < kBatch; ++ss)
#pragma unroll
                        for (int u = 0; u < kPer; ++u)
                            if (s0 + ss < ns) {
                                x0[u] += v[ss][u].x;
                                x1[u] += v[ss][u].y;
                            }
                }
            } else {
#pragma unroll
                for (int u = 0; u < kPer; ++u)
                    if (live[u]) {
                        x0[u] = __ldcg(a.kv + off[u]);
                        x1[u] = __ldcg(a.kv + off[u] + kDP);
                    }
            }
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int it = tid + u * kWorkers;
                if (it >= kItems) continue;
                const int dp = it % (kD / 2), e = (it / (kD / 2)) % kDP, jj = it / (kD / 2 * kDP);
                const int d0 = 2 * dp;
                const float hx0 = __bfloat162float(__float2bfloat16_rn(x0[u]));
                const float hx1 = __bfloat162float(__float2bfloat16_rn(x1[u]));
                const int chunk = jj * 4 + d0 / 8, boff = (d0 % 8) * 2;
                const int lorow = e < kD ? kLoRow + e : kDenLo;   // hi row is e (kDenHi for e = kD)
                *reinterpret_cast<uint32_t*>(bop + sw128_offset(e, chunk) + boff) = pack_bf16x2(hx0, hx1);
                *reinterpret_cast<uint32_t*>(bop + sw128_offset(lorow, chunk) + boff) =
                    pack_bf16x2(x0[u] - hx0, x1[u] - hx1);
            }
            fence_proxy_async_smem();
            mbar_arrive(bfirst);
        };

        // Each group transforms its first tile (Q is not written by pass 1, so it may
        // already have landed), then helps build the first B operand.
        int64_t prev = -1, li = grp;
        float r_prev = 1.f, r_cur = 1.f;
        if (ok && i0 + li < i1) {
            ok = transform(li, r_prev);
            prev = li;
            li += 2;
        }
        if (ok) build_first();
        for (; i0 + li < i1 && ok; li += 2) {
            ok = transform(li, r_cur);
            if (ok) ok = epilogue(prev, r_prev);
            prev = li;
            r_prev = r_cur;
        }
        if (ok && prev >= 0) ok = epilogue(prev, r_prev);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// arrives on, gives up after limit_ns, and records kErrWaitTimeout at `site`.
__global__ void wait_timeout_selftest(uint64_t limit_ns, int site)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_wait(&bar, 0, site, limit_ns);
    }
}

}  // namespace sana
