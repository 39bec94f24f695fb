// Eq. (1) of "Sana: Efficient High-Resolution Image Synthesis with Linear
// Diffusion Transformers", section 2.1 (with the per-head QK-RMSNorm of "SANA 1.5
// ...", section "Model architecture", QK Norm bullet), in ONE launch for short
// sequences (N <= 1024, e.g. the 1024px latent: 32 x 32 tokens).  bf16 in and out,
// fp32 accumulation.
//
// At these sizes the two persistent passes spend most of their time on fixed
// costs: two kernel starts, the partial states' round trip through HBM between
// them, and pass 2 building its operand only after pass 1 has drained.  Here a
// thread-block cluster of S = ceil(N / 128) CTAs (S <= 8) owns one row (b, g) of
// 4 heads; CTA s owns tokens [128 s, 128 s + 128) of it and loads its K, V and Q
// tiles at once.  The hardware schedules a cluster's CTAs together, so they can
// wait for one another at cluster barriers without any spin on global memory.
//
//   1. phi(K) in place (the feature map of Eq. (1) after the QK norm),
//      the normaliser column sums on the CUDA cores, and one UMMA chain
//          D[(h,d), (h',e)] = sum_t phi(K)[t,(h,d)] V[t,(h',e)]   (M=N=128, K=128)
//      whose diagonal blocks are this CTA's partial states (as in pass 1).
//   2. The partial state (4 heads x (D+1) x D fp32) goes to shared memory; the
//      CTA transforms its Q tile while the cluster barrier completes.  CTA s then
//      sums its share of the state's 132 rows (head, e) over the S partials, read
//      from the peers' shared memory in rank order (fixed order: the result is
//      bitwise reproducible and the same in every CTA).  Cluster barrier.
//   3. Every CTA reads the summed rows back from their owners and writes its own
//      B operands (per head 64 rows: the bf16 "hi" parts of the value columns,
//      then their "lo" parts x - bf16(x), so the state keeps ~16 mantissa bits),
//      then per head two UMMAs (M=128, N=64, K=16 each) against phi(Q).  The
//      normaliser phi(Q) . ksum is a 32-term fp32 dot product on the CUDA cores,
//      which frees the TMEM columns it would take: all four heads fit at once.
//      Epilogue O = r num / (r den + eps) written over the Q tile and TMA-stored.
//
// Shared memory (about 99 KB, two CTAs per SM): the K / V tiles (64 KB) become,
// once the state UMMAs have read them, the partial-state export, the summed rows
// and the B operands; the Q tile (32 KB) becomes O.  TMEM: 256 columns, the state
// accumulator in 0..127, then head (pair p, j) in 64 (2 p + j) .. + 63.
//
// TMEM: warp w reads lanes 32 * (w % 4) .. + 31; D row i is lane i.
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

namespace sc {
constexpr int kTok = 128;                          // tokens per CTA (UMMA M of the apply)
constexpr int kMaxCluster = 8;                     // portable cluster size limit
constexpr int kThreads = 256;
constexpr int kHeads = 4;                          // heads per row (the state UMMA's M = 128)
constexpr int kStageTok = 64;                      // K / V tiles: 2 stages of 64 tokens
constexpr int kBoxBytes = kStageTok * 128;         // 64 tokens x 64 channels, bf16
constexpr int kStageBytes = 4 * kBoxBytes;         // [K box 0 | K box 1 | V box 0 | V box 1]
constexpr int kKVBytes = 2 * kStageBytes;          // 64 KB
constexpr int kQBoxBytes = kTok * 128;             // 128 tokens x 64 channels (a head pair)
constexpr int kQBytes = 2 * kQBoxBytes;            // 32 KB
constexpr int kRows = kHeads * kDP;                // state rows (head, e), e = D: normaliser
constexpr int kStateBytes = kRows * kD * 4;        // 16,896
constexpr int kExportOff = 0;                      // this CTA's partial state   (in K / V)
constexpr int kRedOff = 17 * 1024;                 // the rows this CTA summed   (in K / V)
constexpr int kBopOff = 34 * 1024;                 // B operands of the 2 pairs  (in K / V)
constexpr int kN = 64;                             // B rows per head: D hi, then D lo parts
constexpr int kBopBytes = kN * 128;                // one pair, 8 KB
constexpr int kQOff = kKVBytes;
constexpr int kGainOff = kQOff + kQBytes;          // gk[128], gq[128]
constexpr int kKsOff = kGainOff + 2 * kHeads * kD * 4;   // column sums [2 stages][4 heads][32]
constexpr int kOwnOff = kKsOff + 2 * kHeads * kD * 4;    // owning CTA of each state row
constexpr int kKsumOff = kOwnOff + 256;                  // the summed normaliser rows [4][32]
constexpr int kBarOff = kKsumOff + kHeads * kD * 4;
constexpr int kSmemBytes = 1024 + kBarOff + 64;
constexpr int kTmemCols = 256;
static_assert(kExportOff + kStateBytes <= kRedOff && kRedOff + kStateBytes <= kBopOff, "layout");
static_assert(kBopOff % 1024 == 0 && kBopBytes % 1024 == 0, "B operands start on swizzle atoms");
static_assert(kBopOff + 2 * kBopBytes <= kKVBytes, "state areas live in the K / V tiles");
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");
static_assert(kD == 32 && kThreads == 8 * 32, "warp roles assume D = 32 and 8 warps");
}  // namespace sc

struct ScArgs {
    const float* gq;     // gains [C], or nullptr with the norm off
    const float* gk;
    int N, H;
    int S;               // CTAs per cluster: ceil(N / 128) <= 8
    float eps;
    int norm;
};

// grid (S, G, B), cluster (S, 1, 1): blockIdx.x is the CTA's rank in its cluster,
// (blockIdx.z, blockIdx.y) = (b, g).
__global__ void __launch_bounds__(sc::kThreads, 2)
forward_short_cluster(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v,
                      const __grid_constant__ CUtensorMap tmap_o, const ScArgs a)
{
    using namespace sc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* skv = smem;
    uint8_t* sq = smem + kQOff;
    float* sgk = (float*)(smem + kGainOff);
    float* sgq = sgk + kHeads * kD;
    float* kspart = (float*)(smem + kKsOff);
    uint8_t* sown = smem + kOwnOff;
    float* sksum = (float*)(smem + kKsumOff);
    float* expo = (float*)(smem + kExportOff);
    float* red = (float*)(smem + kRedOff);
    uint8_t* bop = smem + kBopOff;
    uint64_t* bar_kv = (uint64_t*)(smem + kBarOff);
    uint64_t* bar_q = bar_kv + 1;
    uint64_t* bar_acc = bar_kv + 2;
    uint64_t* bar_mma = bar_kv + 3;
    uint32_t* tmem_slot = (uint32_t*)(bar_kv + 4);

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int S = a.S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int C = a.H * kD;
    const int tok0 = s * kTok;
    bool ok = true;

    if (tid == 0) {
        mbar_init(bar_kv, 1);
        mbar_init(bar_q, 1);
        mbar_init(bar_acc, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_o);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // Inputs may come from the previous grid: wait for it before any global read.
    pdl_wait_primary();
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_kv, kKVBytes);
        for (int st = 0; st < 2; ++st) {
            uint8_t* sb = skv + st * kStageBytes;
            const int y = tok0 + st * kStageTok;
            tma_load_3d(sb, &tmap_k, bar_kv, g * 128, y, b);
            tma_load_3d(sb + kBoxBytes, &tmap_k, bar_kv, g * 128 + 64, y, b);
            tma_load_3d(sb + 2 * kBoxBytes, &tmap_v, bar_kv, g * 128, y, b);
            tma_load_3d(sb + 3 * kBoxBytes, &tmap_v, bar_kv, g * 128 + 64, y, b);
        }
        mbar_arrive_expect_tx(bar_q, kQBytes);
        tma_load_3d(sq, &tmap_q, bar_q, g * 128, tok0, b);
        tma_load_3d(sq + kQBoxBytes, &tmap_q, bar_q, g * 128 + 64, tok0, b);
    }
    pdl_launch_dependents();
    if (a.norm) {
        const int c = g * 128 + (tid & 127);
        (tid < 128 ? sgk : sgq)[tid & 127] = c < C ? (tid < 128 ? a.gk : a.gq)[c] : 0.f;
    }
    // state rows (head, e) are split over the cluster's CTAs in contiguous ranges
    if (tid < kRows) sown[tid] = (uint8_t)owner_cta(tid, kRows, S);
    const int r0 = s * kRows / S, r1 = (s + 1) * kRows / S;
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ---------------------------------------------------------------- 1. phi(K), state
    {
        // warp w: stage w / 4 (64 tokens), head w % 4; lane l: token rows l, l + 32
        const int st = warp >> 2, hl = warp & 3, h = g * kHeads + hl;
        ok = mbar_wait(bar_kv, 0, 501) && ok;
        uint8_t* const tl[2] = {skv + st * kStageBytes + (hl >> 1) * kBoxBytes,
                                skv + st * kStageBytes + (hl >> 1) * kBoxBytes};
        const int rows[2] = {lane, lane + 32}, ch[2] = {(hl & 1) * 4, (hl & 1) * 4};
        const int t = tok0 + st * kStageTok;
        const bool dead[2] = {!(t + lane < a.N && h < a.H), !(t + lane + 32 < a.N && h < a.H)};
        const float* gg[2] = {sgk + hl * kD, sgk + hl * kD};
        float ks[kD], rr[2];
#pragma unroll
        for (int e = 0; e < kD; ++e) ks[e] = 0.f;
        phi2_inplace_sw128<true>(tl, rows, ch, gg, a.eps, a.norm != 0, dead, rr, ks);
        warp_reduce_scatter32(ks, lane);
        kspart[(st * kHeads + hl) * kD + lane] = ks[0];
        fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) {
        const uint32_t idesc = make_idesc_bf16(128, 128, true, true);
        const uint64_t k0 = make_smem_desc(smem_u32(skv), kBoxBytes, 1024, kSwizzle128B);
        const uint64_t v0 = k0 + (uint64_t)((2 * kBoxBytes) >> 4);
#pragma unroll
        for (int st = 0; st < 2; ++st) {
            const uint64_t so = (uint64_t)((st * kStageBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kStageTok / 16; ++kk)
                umma_bf16_elect(tmem, k0 + so + kk * 128, v0 + so + kk * 128, idesc,
                                !(st == 0 && kk == 0));
        }
        umma_commit_elect(bar_acc);
    }

    // ---------------------------------------------------------------- 2. export, reduce
    // warp w: token row 32 (w % 4) + lane (its TMEM lane quadrant) in the apply;
    // here head w % 4's diagonal block, columns e in [16 (w / 4), + 16)
    const int q4 = warp & 3, jj = warp >> 2;
    const int row = 32 * q4 + lane;
    ok = mbar_wait(bar_acc, 0, 503) && ok;
    tc_fence_after_sync();
    {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q4) << 16) + 32 * q4 + 16 * jj, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) expo[(q4 * kDP + 16 * jj + i) * kD + lane] = v[i];
        if (jj == 0)
            expo[(q4 * kDP + kD) * kD + lane] =
                kspart[q4 * kD + lane] + kspart[(kHeads + q4) * kD + lane];
    }
    tc_fence_before_sync();
    cluster_arrive();
    // phi(Q) while the cluster catches up: heads (pair 0, w / 4) and (pair 1, w / 4)
    // of token row `row`.  The positive per-token factor r of phi(Q) is applied in
    // the epilogue (O = r num' / (r den' + eps)), so the operand holds ReLU(g q).
    float rq[2];
    {
        ok = mbar_wait(bar_q, 0, 502) && ok;
        uint8_t* const tl[2] = {sq, sq + kQBoxBytes};
        const int rows[2] = {row, row}, ch[2] = {jj * 4, jj * 4};
        const int hA = g * kHeads + jj, hB = g * kHeads + 2 + jj;
        const bool dead[2] = {!(tok0 + row < a.N && hA < a.H), !(tok0 + row < a.N && hB < a.H)};
        const float* gg[2] = {sgq + jj * kD, sgq + (2 + jj) * kD};
        phi2_inplace_sw128<false>(tl, rows, ch, gg, a.eps, a.norm != 0, dead, rq, nullptr);
        fence_proxy_async_smem();
    }
    cluster_wait();                                               // every partial is out
    {
        // items: 4 consecutive d of one row this CTA owns; its S partials are summed
        // in rank order
        const uint32_t ex = smem_u32(expo);
        for (int it = tid; it < (r1 - r0) * (kD / 4); it += kThreads) {
            const int r = r0 + (it >> 3), dq = it & 7;
            const uint32_t off = (uint32_t)(r * kD + 4 * dq) * 4;
            float4 v[kMaxCluster];
#pragma unroll
            for (int src = 0; src < kMaxCluster; ++src)
                v[src] = src < S ? ld_cluster_f32x4(map_shared_rank(ex + off, src))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 acc = v[0];
#pragma unroll
            for (int src = 1; src < kMaxCluster; ++src)
                if (src < S) {
                    acc.x += v[src].x;
                    acc.y += v[src].y;
                    acc.z += v[src].z;
                    acc.w += v[src].w;
                }
            *reinterpret_cast<float4*>(red + r * kD + 4 * dq) = acc;
        }
    }
    cluster_arrive();
    cluster_wait();                                               // every row is summed

    // ---------------------------------------------------------------- 3. B operands
    {
        // items: 4 consecutive d of one row, read from the row's owner.  Value rows
        // (e < D) go to the B operand as bf16 hi / lo parts (rows e and D + e); the
        // normaliser row stays fp32 for the epilogue's CUDA-core dot product.
        constexpr int kItems = kRows * (kD / 4);
        constexpr int kPer = (kItems + kThreads - 1) / kThreads;
        const uint32_t rd = smem_u32(red);
        float4 v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int it = tid + u * kThreads;
            const int r = it >> 3, dq = it & 7;
            v[u] = it < kItems ? ld_cluster_f32x4(map_shared_rank(
                                     rd + (uint32_t)(r * kD + 4 * dq) * 4, sown[r]))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int it = tid + u * kThreads;
            if (it >= kItems) continue;
            const int r = it >> 3, dq = it & 7;
            const int j = r / kDP, e = r % kDP;
            const int d0 = 4 * dq;
            if (e == kD) {
                *reinterpret_cast<float4*>(sksum + j * kD + d0) = v[u];
                continue;
            }
            const int chunk = (j & 1) * 4 + d0 / 8, boff = (d0 % 8) * 2;
            uint8_t* dst = bop + (j >> 1) * kBopBytes;
            const float h0 = __bfloat162float(__float2bfloat16_rn(v[u].x));
            const float h1 = __bfloat162float(__float2bfloat16_rn(v[u].y));
            const float h2 = __bfloat162float(__float2bfloat16_rn(v[u].z));
            const float h3 = __bfloat162float(__float2bfloat16_rn(v[u].w));
            *reinterpret_cast<uint2*>(dst + sw128_offset(e, chunk) + boff) =
                make_uint2(pack_bf16x2(h0, h1), pack_bf16x2(h2, h3));
            *reinterpret_cast<uint2*>(dst + sw128_offset(kD + e, chunk) + boff) =
                make_uint2(pack_bf16x2(v[u].x - h0, v[u].y - h1),
                           pack_bf16x2(v[u].z - h2, v[u].w - h3));
        }
        fence_proxy_async_smem();
    }
    cluster_arrive();              // done with the peers' shared memory (waited for at exit)
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    if (warp == 0) {
        // head (p, j) of the row: D[t, n] = sum_d phi(Q)[t, d] Bop_(p,j)[n, d] in
        // columns 64 (2 p + j) .. + 63 (n < D: hi parts of the value columns, n >= D: lo)
        const uint32_t idesc = make_idesc_bf16(128, kN, false, false);
        const uint64_t a0 = make_smem_desc(smem_u32(sq), 16, 1024, kSwizzle128B);
        const uint64_t b0 = make_smem_desc(smem_u32(bop), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint64_t ad = a0 + (uint64_t)((p * kQBoxBytes) >> 4) + 4 * j;
                const uint64_t bd = b0 + (uint64_t)((p * kBopBytes) >> 4) + 4 * j;
                umma_bf16_elect(tmem + kN * (2 * p + j), ad, bd, idesc, false);
                umma_bf16_elect(tmem + kN * (2 * p + j), ad + 2, bd + 2, idesc, true);
            }
        umma_commit_elect(bar_mma);
    }

    // ---------------------------------------------------------------- epilogue
    // head (p, jj) of token row `row`:
    //   O = (hi + lo) r / (r den' + eps),  den' = phi(Q)' . ksum (fp32, CUDA cores)
    ok = mbar_wait(bar_mma, 0, 505) && ok;
    tc_fence_after_sync();
#pragma unroll 1
    for (int p = 0; p < 2; ++p) {
        uint8_t* box = sq + p * kQBoxBytes;
        const float* ksj = sksum + (2 * p + jj) * kD;
        float den = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(box + sw128_offset(row, jj * 4 + c));
            const float4 k0 = *reinterpret_cast<const float4*>(ksj + 8 * c);
            const float4 k1 = *reinterpret_cast<const float4*>(ksj + 8 * c + 4);
            den = fmaf(bf16lo(u.x), k0.x, den); den = fmaf(bf16hi(u.x), k0.y, den);
            den = fmaf(bf16lo(u.y), k0.z, den); den = fmaf(bf16hi(u.y), k0.w, den);
            den = fmaf(bf16lo(u.z), k1.x, den); den = fmaf(bf16hi(u.z), k1.y, den);
            den = fmaf(bf16lo(u.w), k1.z, den); den = fmaf(bf16hi(u.w), k1.w, den);
        }
        const uint32_t ta = tmem + ((uint32_t)(32 * q4) << 16) + kN * (2 * p + jj);
        float hi[kD], lo[kD];
        tmem_ld16(ta, hi);
        tmem_ld16(ta + 16, hi + 16);
        tmem_ld16(ta + kD, lo);
        tmem_ld16(ta + kD + 16, lo + 16);
        tmem_wait_ld();
        const float r = p == 0 ? rq[0] : rq[1];
        const float scale = r * __frcp_rn(fmaf(r, den, a.eps));
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
            *reinterpret_cast<uint4*>(box + sw128_offset(row, jj * 4 + cc)) = w;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tma_store_3d(&tmap_o, sq, g * 128, tok0, b);
        if (g * 128 + 64 < C) tma_store_3d(&tmap_o, sq + kQBoxBytes, g * 128 + 64, tok0, b);
        bulk_commit_group();
        bulk_wait_group_read<0>();         // the tile may go; the writes finish on their own
    }
    cluster_wait();                // no peer still reads this CTA's shared memory
    __syncwarp();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
    (void)ok;
}

}  // namespace sana
