// Tensor-core (tcgen05 + TMA) kernels for the two passes of Eq. (1), "Sana:
// Efficient High-Resolution Image Synthesis with Linear Diffusion Transformers",
// section 2.1, with the per-head QK-RMSNorm of "SANA 1.5 ...", section "Model
// architecture" (QK Norm bullet).  bf16 inputs and outputs, fp32 accumulation.
//
// Both passes are HBM-bound (16.5 flop per byte); the D x (D+1) contractions go
// to the tensor cores only because CUDA-core FMAs cannot keep up with HBM here.
// Both kernels are persistent: one CTA per SM walks a contiguous, balanced range
// of a flat work list, so there is no tail wave and setup is paid once per SM.
//
// Pass 1, kv_reduce_persistent.  Work item = one 64-token stage of one row
// (b, g), g a group of 4 heads (128 channels).  Per stage:
//     D[(h,d), (h',e)] += sum_t phi(K)[t,(h,d)] V[t,(h',e)]       (UMMA M=128, N=128)
//     D[(h,d), 128]    += sum_t phi(K)[t,(h,d)]                   (UMMA N=64, ones)
// and the diagonal blocks h == h' are the state.  TMA brings K and V tiles with the
// 128-byte swizzle, [token][channel]; the transform warps rewrite K in place as
// phi(K) = ReLU(g * k / rms(k)), which makes it the MN-major A operand; V already
// is the MN-major B operand.  At the end of each row segment the epilogue warps
// store the segment's partial state; the last CTA to finish a row (global
// counter) sums that row's partials in CTA order into the final state, so the
// result is bitwise reproducible.
//
// Pass 2, apply_persistent.  Work item = one 128-token tile of one row (b, p), p a
// pair of heads (64 channels).  A builder warp turns the fp32 state of the row into
// the B operand per head (n = value column e or the normaliser, k = d; bf16 hi and
// lo parts, so the state keeps ~16 mantissa bits); the workers rewrite the Q tile
// in place as phi(Q) (K-major A operand); UMMA M=128 N=48 (K=16 x 2 x {hi, lo})
//     D[t, e] = sum_d phi(Q)[t,d] S[d,e],  e < 32;   D[t, 32] = sum_d phi(Q)[t,d] S[d,32]
// and the workers form O = D[:, :32] * (1 / (D[:, 32] + eps)), write it over the
// tile and TMA-store it.  Only the builder warp reads what pass 1 wrote, so under
// programmatic dependent launch the Q stream starts while pass 1 finishes.
//
// TMEM: warp w reads lanes 32 * (w % 4) .. + 31; D row i is lane i.
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"

namespace sana {

// The feature map on 32 values held as 4 swizzled 16-byte chunks of row `row`,
// starting at chunk `chunk0`, rewritten in place as bf16.  g points at the
// head's 32 gains in shared memory (ignored with the norm off).
//   scale_by_rms: phi = ReLU(g * x * r) with r = rsqrt(mean(x^2) + eps)
//   otherwise   : ReLU(g * x) is written and r is returned for the caller to
//                 apply later (it is a positive per-token factor).
//   norm off    : ReLU(x); returns 1.
//   zero        : writes zeros (rows past N, heads past H); returns 1.
template <bool kScaleByRms>
__device__ __forceinline__ float phi_inplace_sw128(uint8_t* tile, int row, int chunk0,
                                                   const float* g, float eps, bool norm,
                                                   bool zero) {
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
        if (kScaleByRms) {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = fmaxf(g[i] * (x[i] * r), 0.f);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = fmaxf(g[i] * x[i], 0.f);
        }
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
    }
    return kScaleByRms ? 1.f : r;
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
    return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// ============================================================================ pass 1
namespace p1 {
constexpr int kGroupHeads = 4;                     // heads per row (UMMA M = 128)
constexpr int kRingBytes = 192 * 1024;             // TMA ring: K and V stages
constexpr int kOnesBytes = 16 * 128;               // 16 token rows x 64 columns
constexpr int kAccStride = 256;                    // TMEM columns between the two accumulators
constexpr int kTmemCols = 512;
constexpr int kTransformWarps = 8;                 // two groups of 4, alternating stages
constexpr int kEpilogueWarps = 4;
constexpr int kThreads = 32 * (2 + kTransformWarps + kEpilogueWarps);
constexpr int kGainCache = 4096;                   // channels whose gains live in smem
constexpr int kSmemBytes = 1024 + kRingBytes + kOnesBytes + kGainCache * 4 + 1024;

// Stage geometry for kStageTok tokens per stage: boxes of kStageTok tokens x 64
// channels, [K box 0 | K box 1 | V box 0 | V box 1], as many stages as fit the ring.
template <int kStageTok>
struct Stage {
    static constexpr int kBoxBytes = kStageTok * 128;
    static constexpr int kBytes = 4 * kBoxBytes;
    static constexpr int kCount = kRingBytes / kBytes;
    static constexpr int kItemsPerThread = kStageTok * kGroupHeads / 128;
    static_assert(kStageTok % 16 == 0 && kStageTok <= 256, "stage rows");
    // The two transform groups take alternate stages; with an even slot count
    // every slot belongs to one group, so each mbarrier phase is awaited in order
    // (an odd count would let a group test a slot's next phase before the current
    // one completed).
    static_assert(kCount >= 2 && kCount % 2 == 0, "ring slots must be even");
};
}  // namespace p1

struct P1Args {
    const float* gk;     // gains [C], or nullptr with the norm off
    float* part;         // partial states [B][H][Smax][D][D+1]
    float* kv;           // final states [B][H][D][D+1]
    int* counters;       // [B * G], zero on entry
    int64_t T;           // work items: B * G rows x R stages
    int N, H, G, R, Smax, P;
    float eps;
    int norm;
};

template <int kStageTok>
__global__ void __launch_bounds__(p1::kThreads, 1)
kv_reduce_persistent(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const P1Args a)
{
    using namespace p1;
    constexpr int kBoxBytes = Stage<kStageTok>::kBoxBytes;
    constexpr int kStageBytes = Stage<kStageTok>::kBytes;
    constexpr int kStages = Stage<kStageTok>::kCount;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* ones = stages + kRingBytes;
    float* sgain = (float*)(ones + kOnesBytes);
    uint64_t* full = (uint64_t*)(sgain + kGainCache);
    uint64_t* aready = full + kStages;
    uint64_t* empty = aready + kStages;
    uint64_t* accfull = empty + kStages;
    uint64_t* accempty = accfull + 2;
    uint64_t* drain = accempty + 2;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    int* last_flag = (int*)(tmem_slot + 1);

    pdl_launch_dependents();   // the apply pass may take each SM as soon as this CTA leaves

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
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    for (int i = threadIdx.x; i < kOnesBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(ones)[i] = make_uint4(0, 0, 0, 0);
    if (a.norm)
        for (int i = threadIdx.x; i < C; i += blockDim.x) sgain[i] = a.gk[i];
    __syncthreads();
    if (threadIdx.x < 16)   // the normaliser operand: column 0 of every row is 1.0
        *reinterpret_cast<uint16_t*>(ones + sw128_offset(threadIdx.x, 0)) = 0x3F80;
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
        // ------------------------------------------------ TMA producer
        if (lane == 0 && ok) {
            int64_t last = -1;
            for (int64_t li = 0; i0 + li < i1; ++li) {
                const int st = (int)(li % kStages);
                if (li >= kStages) ok = mbar_wait(&empty[st], (uint32_t)((li / kStages) - 1) & 1, 301);
                if (!ok) break;
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.G), g = (int)(r % a.G);
                uint8_t* sb = stages + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                const int x = g * 128, y = t * kStageTok;
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
        // ------------------------------------------------ UMMA issuer
        if (lane == 0 && ok) {
            const uint32_t idesc_v = make_idesc_bf16(128, 128, true, true);
            const uint32_t idesc_1 = make_idesc_bf16(128, 64, true, true);
            const uint64_t ones_desc =
                make_smem_desc(smem_u32(ones), kBoxBytes, 1024, kSwizzle128B);
            int seg = 0;
            for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
                const int64_t i = i0 + li;
                const int t = (int)(i % a.R), st = (int)(li % kStages);
                const bool first = (li == 0) || (t == 0);
                const bool lastst = (i + 1 == i1) || (t == a.R - 1);
                const int abuf = seg & 1;
                if (first && seg >= 2)
                    ok = mbar_wait(&accempty[abuf], (uint32_t)((seg >> 1) - 1) & 1, 303);
                if (ok) ok = mbar_wait(&aready[st], (uint32_t)(li / kStages) & 1, 304);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d = tmem + abuf * kAccStride;
                const uint32_t kb = smem_u32(stages + st * kStageBytes);
                const uint32_t vb = kb + 2 * kBoxBytes;
#pragma unroll
                for (int kk = 0; kk < kStageTok / 16; ++kk) {
                    const uint64_t ad = make_smem_desc(kb + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
                    const uint64_t bd = make_smem_desc(vb + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
                    const bool acc = !(first && kk == 0);
                    umma_bf16(d, ad, bd, idesc_v, acc);
                    umma_bf16(d + 128, ad, ones_desc, idesc_1, acc);
                }
                umma_commit(&empty[st]);
                if (lastst) {
                    umma_commit(&accfull[abuf]);
                    ++seg;
                }
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 305);
        }
    } else if (warp < 2 + kTransformWarps) {
        // ------------------------------------------------ phi(K) in place
        // Two groups of 4 warps take alternate stages, so two stages are in the
        // transform at once.  Within a stage, item idx = (head, token row) with the
        // row fastest, so each quarter warp touches 8 consecutive swizzled rows.
        const int wt = threadIdx.x - 64;                 // 0..255
        const int grp = wt >> 7;                         // stages with li % 2 == grp
        const int gt = wt & 127;
        for (int64_t li = grp; i0 + li < i1 && ok; li += 2) {
            const int st = (int)(li % kStages);
            ok = mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 306);
            if (!ok) break;
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), g = (int)(r % a.G);
#pragma unroll
            for (int it = 0; it < Stage<kStageTok>::kItemsPerThread; ++it) {
                const int idx = gt + it * 128;
                const int row = idx % kStageTok, hl = idx / kStageTok;
                const int h = g * kGroupHeads + hl;
                const bool live = (t * kStageTok + row < a.N) && (h < a.H);
                phi_inplace_sw128<true>(stages + st * kStageBytes + (hl >> 1) * kBoxBytes, row,
                                        (hl & 1) * 4, sgain + (live ? h : 0) * kD, a.eps,
                                        a.norm != 0, !live);
            }
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
        }
    } else {
        // ------------------------------------------------ segment epilogue + combine
        const int et = threadIdx.x - 32 * (2 + kTransformWarps);   // 0..127
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
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + abuf * kAccStride;
            float v[32], ks;
            tmem_ld16(ta + 32 * q, v);
            tmem_ld16(ta + 32 * q + 16, v + 16);
            tmem_ld1(ta + 128, &ks);
            tmem_wait_ld();
            tc_fence_before_sync();
            mbar_arrive(&accempty[abuf]);
            ++seg;

            const int64_t r = i / a.R;
            const int b = (int)(r / a.G), g = (int)(r % a.G);
            const int64_t first_owner = owner_cta(r * a.R, a.T, a.P);
            const int nslots = (int)(owner_cta(r * a.R + a.R - 1, a.T, a.P) - first_owner + 1);
            const int slot = (int)(c - first_owner);
            const int h = g * kGroupHeads + q;
            if (h < a.H) {
                float* o = a.part + (((size_t)b * a.H + h) * a.Smax + slot) * kStateFloats + lane * kDP;
#pragma unroll
                for (int e = 0; e < kD; ++e) o[e] = v[e];
                o[kD] = ks;
            }
            __threadfence();
            named_barrier_sync(1, 32 * kEpilogueWarps);
            if (et == 0) *last_flag = (atomicAdd(&a.counters[r], 1) == nslots - 1);
            named_barrier_sync(1, 32 * kEpilogueWarps);
            if (*last_flag) {
                __threadfence();
                // sum the row's partial slots in slot order; float4 lanes, all loads of
                // a slot issued before any add so they overlap
                constexpr int kVec = kStateFloats / 4;                    // 264 float4 per head
                for (int base = et; base < kGroupHeads * kVec; base += 3 * 32 * kEpilogueWarps) {
                    float4 acc[3];
                    int hh[3], e4[3];
#pragma unroll
                    for (int u = 0; u < 3; ++u) {
                        const int idx = base + u * 32 * kEpilogueWarps;
                        hh[u] = g * kGroupHeads + idx / kVec;
                        e4[u] = idx % kVec;
                        if (idx >= kGroupHeads * kVec) hh[u] = a.H;       // past the group
                        acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    for (int s = 0; s < nslots; s += 2) {      // two slots in flight
                        float4 x[2][3];
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2)
#pragma unroll
                            for (int u = 0; u < 3; ++u)
                                if (hh[u] < a.H && s + w2 < nslots)
                                    x[w2][u] = __ldcg(reinterpret_cast<const float4*>(
                                                   a.part + (((size_t)b * a.H + hh[u]) * a.Smax +
                                                             s + w2) * kStateFloats) + e4[u]);
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2)
#pragma unroll
                            for (int u = 0; u < 3; ++u)
                                if (hh[u] < a.H && s + w2 < nslots) {
                                    acc[u].x += x[w2][u].x; acc[u].y += x[w2][u].y;
                                    acc[u].z += x[w2][u].z; acc[u].w += x[w2][u].w;
                                }
                    }
#pragma unroll
                    for (int u = 0; u < 3; ++u)
                        if (hh[u] < a.H)
                            reinterpret_cast<float4*>(a.kv + ((size_t)b * a.H + hh[u]) * kStateFloats)
                                [e4[u]] = acc[u];
                }
            }
            named_barrier_sync(1, 32 * kEpilogueWarps);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ============================================================================ pass 2
namespace p2 {
constexpr int kTileTok = 128;                      // UMMA M
constexpr int kPairHeads = 2;                      // 64 channels = one swizzled row
constexpr int kTileBytes = kTileTok * 128;         // 16 KB
constexpr int kStages = 10;
constexpr int kN = 48;                             // 32 value columns, normaliser, padding
constexpr int kBopBytes = kN * 128;                // per head: rows n, [hi d0..31 | lo d0..31]
constexpr int kBopSetBytes = kPairHeads * kBopBytes;
constexpr int kBopRing = 2;
constexpr int kBufCols = kPairHeads * kN;          // 96 TMEM columns per tile
constexpr int kTmemBufs = 4;
constexpr int kTmemCols = 512;
constexpr int kWorkerWarps = 8;                    // two groups of 4, alternating tiles
static_assert(kStages % 2 == 0, "each ring slot must belong to one worker group");
constexpr int kThreads = 32 * (3 + kWorkerWarps);
constexpr int kGainCache = 4096;
constexpr int kStateStageBytes = kPairHeads * kStateFloats * 4;   // fp32 states of a pair
constexpr int kSmemBytes = 1024 + kStages * kTileBytes + kBopRing * kBopSetBytes +
                           kStateStageBytes + kGainCache * 4 + 1024;
}  // namespace p2

struct P2Args {
    const float* kv;     // states [B][H][D][D+1] (written by pass 1 when chained)
    const float* gq;     // gains [C] or nullptr
    int64_t T;           // work items: B * Pp rows x R tiles
    int N, H, Pp, R, P;
    float eps;
    int norm;
};

__global__ void __launch_bounds__(p2::kThreads, 1)
apply_persistent(const __grid_constant__ CUtensorMap tmap_q,
                 const __grid_constant__ CUtensorMap tmap_o, const P2Args a)
{
    using namespace p2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* bop = stages + kStages * kTileBytes;
    float* sstate = (float*)(bop + kBopRing * kBopSetBytes);
    float* sgain = sstate + kPairHeads * kStateFloats;
    uint64_t* full = (uint64_t*)(sgain + kGainCache);
    uint64_t* aready = full + kStages;
    uint64_t* mmadone = aready + kStages;
    uint64_t* empty = mmadone + kStages;
    uint64_t* tfree = empty + kStages;
    uint64_t* bfull = tfree + kTmemBufs;
    uint64_t* bempty = bfull + kBopRing;
    uint64_t* drain = bempty + kBopRing;
    uint64_t* sready = drain + 1;
    uint32_t* tmem_slot = (uint32_t*)(sready + 1);

    const int64_t c = blockIdx.x;
    const int64_t i0 = range_begin(c, a.T, a.P), i1 = range_begin(c + 1, a.T, a.P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.H * kD;                      // at most kGainCache (checked on the host)

    if (threadIdx.x == 0) {
        mbar_init(sready, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], 128);
            mbar_init(&mmadone[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < kTmemBufs; ++i) mbar_init(&tfree[i], 128);
        for (int i = 0; i < kBopRing; ++i) {
            mbar_init(&bfull[i], 32);
            mbar_init(&bempty[i], 1);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_o);
    }
    if (a.norm)
        for (int i = threadIdx.x; i < C; i += blockDim.x) sgain[i] = a.gq[i];
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
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
        // ------------------------------------------------ UMMA issuer
        if (lane == 0 && ok) {
            const uint32_t idesc = make_idesc_bf16(128, kN, false, false);
            int seg = 0;
            for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
                const int64_t i = i0 + li;
                const int t = (int)(i % a.R), st = (int)(li % kStages);
                const bool first = (li == 0) || (t == 0);
                const bool lastt = (i + 1 == i1) || (t == a.R - 1);
                const int rb = seg & 1, tb = (int)(li % kTmemBufs);
                if (first) ok = mbar_wait(&bfull[rb], (uint32_t)(seg >> 1) & 1, 403);
                if (ok) ok = mbar_wait(&aready[st], (uint32_t)(li / kStages) & 1, 404);
                if (ok && li >= kTmemBufs)
                    ok = mbar_wait(&tfree[tb], (uint32_t)((li / kTmemBufs) - 1) & 1, 405);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t ab = smem_u32(stages + st * kTileBytes);
                const uint32_t bb0 = smem_u32(bop + rb * kBopSetBytes);
#pragma unroll
                for (int j = 0; j < kPairHeads; ++j) {
                    const uint32_t d = tmem + tb * kBufCols + j * kN;
                    const uint32_t bb = bb0 + j * kBopBytes;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t ad = make_smem_desc(ab + j * 64 + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t hi = make_smem_desc(bb + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t lo = make_smem_desc(bb + 64 + kk * 32, 16, 1024, kSwizzle128B);
                        umma_bf16(d, ad, hi, idesc, kk > 0);
                        umma_bf16(d, ad, lo, idesc, true);
                    }
                }
                umma_commit(&mmadone[st]);
                if (lastt) {
                    umma_commit(&bempty[rb]);
                    ++seg;
                }
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 406);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ B operand builder
        // Per row segment: one bulk copy brings the pair's fp32 states into smem,
        // then the 32 lanes write the swizzled bf16 hi/lo operand from there.
        int seg = 0;
        for (int64_t li = 0; i0 + li < i1 && ok; ++li) {
            const int64_t i = i0 + li;
            if (!(li == 0 || i % a.R == 0)) continue;              // not a segment start
            const int rb = seg & 1;
            if (seg >= 2) ok = mbar_wait(&bempty[rb], (uint32_t)((seg >> 1) - 1) & 1, 407);
            if (!ok) break;
            if (seg == 0) pdl_wait_primary();                     // the states come from pass 1
            const int64_t r = i / a.R;
            const int b = (int)(r / a.Pp), p = (int)(r % a.Pp);
            const int nh = min(kPairHeads, a.H - p * kPairHeads);
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)(nh * kStateFloats * 4);
                mbar_arrive_expect_tx(sready, bytes);
                bulk_load(sstate, a.kv + ((size_t)b * a.H + p * kPairHeads) * kStateFloats, bytes,
                          sready);
            }
            ok = mbar_wait(sready, (uint32_t)seg & 1, 410);
            if (!ok) break;
            uint8_t* dst = bop + rb * kBopSetBytes;
            for (int idx = lane; idx < kPairHeads * kN * 8; idx += 32) {
                const int j = idx / (kN * 8), rem = idx % (kN * 8), n = rem >> 3, ch = rem & 7;
                const float* src = sstate + j * kStateFloats;
                float vals[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int dd = (ch & 3) * 8 + u;
                    const float x = (j < nh && n <= kD) ? src[dd * kDP + n] : 0.f;
                    const float hi = __bfloat162float(__float2bfloat16_rn(x));
                    vals[u] = (ch < 4) ? hi : (x - hi);
                }
                uint4 w;
                w.x = pack_bf16x2(vals[0], vals[1]);
                w.y = pack_bf16x2(vals[2], vals[3]);
                w.z = pack_bf16x2(vals[4], vals[5]);
                w.w = pack_bf16x2(vals[6], vals[7]);
                *reinterpret_cast<uint4*>(dst + j * kBopBytes + sw128_offset(n, ch)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();                                         // sstate is reused next segment
            mbar_arrive(&bfull[rb]);
            ++seg;
        }
    } else {
        // ------------------------------------------------ phi(Q), epilogue, TMA store
        const int wi = warp - 3;                          // 0..7
        const int grp = wi >> 2;                          // tiles with li % 2 == grp
        const int gt = (wi & 3) * 32 + lane;              // 0..127 within the group
        const int q = warp & 3;                           // TMEM lane quadrant
        const int row = 32 * q + lane;                    // token row of the tile

        // The per-token factor r = rsqrt(mean(q^2) + eps) of phi(Q) is positive, so it
        // is left out of the A operand and applied in the epilogue:
        //   O = (r num') / (r den' + eps),  num', den' computed with ReLU(g * q).
        auto transform = [&](int64_t li, float* rq) -> bool {
            const int st = (int)(li % kStages);
            if (!mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 408)) return false;
            const int64_t i = i0 + li, r = i / a.R;
            const int t = (int)(i % a.R), p = (int)(r % a.Pp);
            uint8_t* tile = stages + st * kTileBytes;
            const bool row_live = t * kTileTok + row < a.N;
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                const int h = p * kPairHeads + j;
                const bool live = row_live && h < a.H;
                rq[j] = phi_inplace_sw128<false>(tile, row, j * 4, sgain + (live ? h : 0) * kD,
                                                 a.eps, a.norm != 0, !live);
            }
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
            return true;
        };
        auto epilogue = [&](int64_t li, const float* rq) -> bool {
            const int st = (int)(li % kStages), tb = (int)(li % kTmemBufs);
            if (!mbar_wait(&mmadone[st], (uint32_t)(li / kStages) & 1, 409)) return false;
            tc_fence_after_sync();
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * kBufCols;
            float v[kPairHeads][kD + 1];
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                tmem_ld16(ta + j * kN, v[j]);
                tmem_ld16(ta + j * kN + 16, v[j] + 16);
                tmem_ld1(ta + j * kN + kD, v[j] + kD);
            }
            tmem_wait_ld();
            tc_fence_before_sync();
            mbar_arrive(&tfree[tb]);
            uint8_t* tile = stages + st * kTileBytes;
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                const float scale = rq[j] * __frcp_rn(fmaf(rq[j], v[j][kD], a.eps));
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 w;
                    w.x = pack_bf16x2(v[j][8 * cc + 0] * scale, v[j][8 * cc + 1] * scale);
                    w.y = pack_bf16x2(v[j][8 * cc + 2] * scale, v[j][8 * cc + 3] * scale);
                    w.z = pack_bf16x2(v[j][8 * cc + 4] * scale, v[j][8 * cc + 5] * scale);
                    w.w = pack_bf16x2(v[j][8 * cc + 6] * scale, v[j][8 * cc + 7] * scale);
                    *reinterpret_cast<uint4*>(tile + sw128_offset(row, j * 4 + cc)) = w;
                }
            }
            fence_proxy_async_smem();
            named_barrier_sync(1 + grp, 128);
            if (gt == 0) {
                const int64_t i = i0 + li, r = i / a.R;
                const int t = (int)(i % a.R), b = (int)(r / a.Pp), p = (int)(r % a.Pp);
                tma_store_3d(&tmap_o, tile, p * 64, t * kTileTok, b);
                bulk_commit_group();
                bulk_wait_group_read<1>();                // this group's previous store has read smem
                if (li >= 2) mbar_arrive(&empty[(li - 2) % kStages]);
            }
            return true;
        };

        int64_t prev = -1;
        float r_prev[kPairHeads] = {1.f, 1.f}, r_cur[kPairHeads];
        for (int64_t li = grp; i0 + li < i1 && ok; li += 2) {
            ok = transform(li, r_cur);
            if (ok && prev >= 0) ok = epilogue(prev, r_prev);
            prev = li;
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) r_prev[j] = r_cur[j];
        }
        if (ok && prev >= 0) ok = epilogue(prev, r_prev);
        if (gt == 0) bulk_wait_group<0>();
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
