// Device-side building blocks of the AWQ search library (sm_100a only):
//   * the quantizer arithmetic of the per-layer scale search, written once and
//     used by every kernel that evaluates it (group parameters, the search
//     producer, the standalone dequantizer and the packer), so that all of them
//     produce bit-identical codes;
//   * thin inline-PTX wrappers for mbarriers, TMA and the tcgen05 tensor core.
//
// Sources (web pages): [QAS-QA] "Как работает quantization-aware scaling в AWQ
// для защиты важных весов?" §5, §9; [AWQ-note] "AWQ: Activation-Aware Weight
// Quantization For On-Device LLM Compression AND Acceleration", "Measures";
// [AWQ-wiki] "AWQ" (French), "Fondements techniques".
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace awq {

// ---------------------------------------------------------------------------
// Device error word (read and cleared by awq_get_status on the host).  The
// library is a single translation unit, so the definition lives here.
// ---------------------------------------------------------------------------
enum : unsigned { kDevErrTimeout = 1u, kDevErrBadAlpha = 2u, kDevErrBadScale = 4u, kDevErrNotPD = 8u };
__device__ unsigned g_dev_error = 0;

// ---------------------------------------------------------------------------
// Quantizer arithmetic.  Every binary32 step is an explicit round-to-nearest
// intrinsic so the compiler cannot contract or reorder it.
// ---------------------------------------------------------------------------

// 1.5 * 2^23: for |x| <= 2^22, RN32(x + kMagic) = kMagic + rint(x) (ties to
// even, because kMagic is even and the spacing of binary32 there is 1).
constexpr float kMagic = 12582912.0f;
constexpr float kMinScale = 5.9604644775390625e-8f;   // 2^-24, smallest fp16 subnormal
constexpr float kMaxScale = 65504.0f;                  // largest finite fp16

// Per-(row, group) quantizer parameters derived from the group's min and max of
// w' = RN32(w*s) ([QAS-QA] §9: zero_point = True, q_group_size, w_bit):
//   scale = RN32(RN32(mx - mn) / qmax), sh = RN16(clamp(scale, 2^-24, 65504)),
//   r = RN32(1/sh), z = RN16(sat(rint(-mn * r))),
// i.e. zero = round(-min/scale), not clamped to the codes: it is saturated to
// +-65504 and rounded to fp16 because the zeros are stored in fp16, and that
// stored value is the z the codes and W_hat use.  Every product inside rint is
// exact (rint is the only rounding of w'/scale).  RN32(x + kMagic) with x an
// exact product is kMagic + rint(x) for |x| <= 2^22 and is monotone in x, so
// one FMA with kMagic evaluates rint of an exact product, and clamping in that
// shifted domain clamps the code (|z| <= 65504 keeps kMagic - z and
// kMagic + qmax - z inside [2^23, 2^24), where binary32 spacing is 1).
// `clamp` records whether any code of the group needs clamping:
// rint(mn r) + z < 0 or rint(mx r) + z > qmax.  The rounding is monotone in w',
// so when neither end needs it no element of the group does.
struct QParams {
    float r;     // reciprocal of the stored fp16 scale
    float sh;    // the stored fp16 scale, as binary32
    float z;     // zero point: an fp16 integer value in [-65504, 65504] (never -0)
    bool clamp;  // some code of the group leaves [0, qmax] before clamping
};

constexpr float kZeroLo = 12517408.0f;   // kMagic - 65504
constexpr float kZeroHi = 12648416.0f;   // kMagic + 65504

// Group parameters from the group's range [mn, mx] of w' = RN32(w s).
//   asymmetric: scale = RN32(RN32(mx - mn) / qmax), z = RN16(sat(rint(-mn r)))
//   symmetric (sym): scale = RN32(max(-mn, mx) / (2^(b-1) - 1)), z = 2^(b-1)
//     with qmax = 2^b - 1, so 2^(b-1) = (qmax + 1) / 2
// then sh = RN16(clamp(scale)), r = RN32(1 / sh).
__device__ __forceinline__ QParams make_qparams(float mn, float mx, float qmax, bool sym = false) {
    QParams p;
    const float mid = __fmul_rn(0.5f, __fadd_rn(qmax, 1.0f));
    float scale = sym ? __fdiv_rn(fmaxf(-mn, mx), __fsub_rn(mid, 1.0f)) : __fdiv_rn(__fsub_rn(mx, mn), qmax);
    scale = fminf(fmaxf(scale, kMinScale), kMaxScale);
    p.sh = __half2float(__float2half_rn(scale));
    p.r = __frcp_rn(p.sh);
    if (sym) {
        p.z = mid;
    } else {
        // vz - kMagic is exact and +0 when vz == kMagic; saturating in the
        // shifted domain also covers |mn r| > 2^22, where vz is no longer
        // kMagic + rint but still lies beyond the saturation bound.
        const float vz = __fmaf_rn(-mn, p.r, kMagic);
        p.z = __half2float(__float2half_rn(__fsub_rn(fminf(fmaxf(vz, kZeroLo), kZeroHi), kMagic)));
    }
    const float vmn = __fmaf_rn(mn, p.r, kMagic);
    const float vmx = __fmaf_rn(mx, p.r, kMagic);
    p.clamp = (vmn < __fsub_rn(kMagic, p.z)) || (vmx > __fadd_rn(kMagic, __fsub_rn(qmax, p.z)));
    return p;
}

// Compact 8-byte form kept in the search workspace: r as binary32, then the
// fp16 scale, whose sign bit carries the clamp flag (the scale is positive),
// and the fp16 zero point (so one half2 -> float2 conversion unpacks both).
__device__ __forceinline__ uint2 pack_qparams(const QParams &p) {
    const uint32_t shb = __half_as_ushort(__float2half_rn(p.sh)) | (p.clamp ? 0x8000u : 0u);
    const uint32_t zb = __half_as_ushort(__float2half_rn(p.z));
    return make_uint2(__float_as_uint(p.r), shb | (zb << 16));
}
__device__ __forceinline__ QParams unpack_qparams(uint2 v) {
    QParams p;
    p.r = __uint_as_float(v.x);
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
    p.sh = fabsf(f.x);
    p.z = f.y;
    p.clamp = (v.y & 0x8000u) != 0;
    return p;
}

// Three-input minimum / maximum (sm_100).
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed binary32 pair arithmetic (sm_100 FMUL2/FFMA2) through the CUDA
// builtins with round-to-nearest-even per component.  Each multiply and add must round exactly
// once where the quantizer's definition says so; the library is built with
// -fmad=false so that no multiply-add pair is contracted behind our back, and
// every intended fusion is written as fma2_rn / __fmaf_rn.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Quantize-dequantize-unscale of two neighbouring weights in packed binary32
// pairs, as the search producer evaluates it:
//   v = RN32(w' r + kMagic) = kMagic + rint(w' r)      (w' = RN32(w s), one FMA)
//   v clamped to [kMagic - z, kMagic + qmax - z]        (only when `clamp`)
//   (q - z) sh = RN32(v sh - kMagic sh)                  (exact, one FMA)
//   w_hat = RN16(RN32(((q - z) sh) rs))
// Clamping after the shifted rint equals clamping the code, because the
// shifted rint is monotone in w'.  A caller may pass clamp = false only when
// make_qparams found that no code of the group needs it.
struct QPair {
    float2 r, magic, sh, nmsh;
    float vlo, vhi;
};
__device__ __forceinline__ QPair make_qpair(const QParams &p, float qmax) {
    QPair q;
    q.r = make_float2(p.r, p.r);
    q.magic = make_float2(kMagic, kMagic);
    q.sh = make_float2(p.sh, p.sh);
    const float nm = __fmul_rn(-kMagic, p.sh);
    q.nmsh = make_float2(nm, nm);
    q.vlo = __fsub_rn(kMagic, p.z);
    q.vhi = __fadd_rn(kMagic, __fsub_rn(qmax, p.z));
    return q;
}
template <bool kClamp>
__device__ __forceinline__ __half2 dequant_unscale_pair(float2 w, float2 s, float2 rs, const QPair &q) {
    float2 v = fma2_rn(mul2_rn(w, s), q.r, q.magic);
    if (kClamp) {
        v.x = fminf(fmaxf(v.x, q.vlo), q.vhi);
        v.y = fminf(fmaxf(v.y, q.vlo), q.vhi);
    }
    return __float22half2_rn(mul2_rn(fma2_rn(v, q.sh, q.nmsh), rs));
}

// ---------------------------------------------------------------------------
// Small PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Streaming 16-byte load that does not allocate in L1 (read-once data).
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Sixteen streaming 16-byte loads at p, p + stride, ..., p + 15 stride (bytes),
// issued back to back from one asm statement, so all sixteen are in flight
// before any result is used.
__device__ __forceinline__ void ldg_stream_v4x16(const void *p, int64_t stride, uint4 (&v)[16]) {
    uint32_t r[64];
    asm volatile(
        "{\n\t.reg .b64 a;\n\t"
        "mov.b64 a, %64;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%4, %5, %6, %7}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%8, %9, %10, %11}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%12, %13, %14, %15}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%16, %17, %18, %19}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%20, %21, %22, %23}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%24, %25, %26, %27}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%28, %29, %30, %31}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%32, %33, %34, %35}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%36, %37, %38, %39}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%40, %41, %42, %43}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%44, %45, %46, %47}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%48, %49, %50, %51}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%52, %53, %54, %55}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%56, %57, %58, %59}, [a];\n\t"
        "add.s64 a, a, %65;\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%60, %61, %62, %63}, [a];\n\t"
        "}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "l"(p), "l"(stride));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
}

// ----- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `hint_ns` elapse, instead of spinning on the barrier.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false (after raising the device timeout flag and the
// CTA's abort flag) when the phase does not complete within about `limit_ns`,
// or when another role of the CTA has already aborted.  Never traps.  Waiting
// threads are suspended by the hardware between polls (kSuspend; otherwise
// they poll) and may also sleep `sleep_ns` between polls; the abort flag and
// the clock are checked only every 16 polls to keep a long wait cheap in
// issue slots.
template <bool kSuspend = true>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                  uint64_t limit_ns, uint32_t sleep_ns = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
        if (kSuspend ? mbar_try_wait_hint(bar, parity, 20000u) : mbar_try_wait(bar, parity)) return true;
        if (sleep_ns) __nanosleep(sleep_ns);
        if ((n & 15u) == 0) {
            if (*abort_flag) return false;
            const uint64_t now = global_timer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(&g_dev_error, kDevErrTimeout);
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
template <bool kSuspend = true>
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                               uint64_t limit_ns, uint32_t sleep_ns = 0) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_bounded<kSuspend>(bar, parity, abort_flag, limit_ns, sleep_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    return ok != 0;
}

// ----- cluster (CTA pair) helpers ------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
// Arrive (release at cluster scope) on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Cluster-wide barrier; the non-.aligned form, since it follows role code in
// which the lanes of a warp diverge.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// ----- TMA ------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int32_t c0,
                                            int32_t c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}
// 2-D tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar_cluster` is a shared::cluster
// address): the form a CTA pair uses to feed one tcgen05 cta_group::2 MMA.
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const void *tmap, int32_t c0, int32_t c1,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
// Plain (non-tensor) bulk copy global -> this CTA's shared memory; addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Asynchronous global -> shared copies of 16 (L2 only) or 4 bytes, and the
// arrive that fires on `bar` once all of this thread's earlier ones landed
// (.noinc: the barrier's expected count includes these arrivals).
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// One 16-byte shared-memory store (a single 128-bit access per thread).
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core reads operands through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----- tcgen05 --------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ----- tcgen05, CTA pair (cta_group::2) -------------------------------------
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair MMA (issued by the leader CTA only): D (+)= A * B^T with M = 256 split
// over the two CTAs' shared memory (same offsets) and B's N rows likewise.
__device__ __forceinline__ void mma_f16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at the same offset in every CTA of `cta_mask`
// when the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 64 consecutive fp32 columns: thread i of the warp receives lane
// (warp quadrant base + i), columns col .. col+63.  The load and its
// tcgen05.wait::ld sit in ONE asm statement: the destination registers of an
// asynchronous tcgen05.ld are undefined until the wait, and separate
// statements would let the compiler schedule their uses above the wait.
__device__ __forceinline__ void tmem_ld_32x32b_x32_sync(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_32x32b_x64_sync(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzled canonical layout: rows of 64 fp16 (128 B), 8-row groups
// 1024 B apart, 16-byte chunks XOR-permuted by (row mod 8).  The tile base
// must be 1024-byte aligned; advancing `saddr` by 32 B steps through K = 16
// slices inside the 128-byte row.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address / 16
    d |= (uint64_t)1u << 16;                    // leading byte offset (unused when swizzled)
    d |= (uint64_t)(1024u >> 4) << 32;          // stride byte offset: 8 rows * 128 B
    d |= (uint64_t)1u << 46;                    // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                    // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor of tcgen05.mma.kind::f16: fp32 accumulator, fp16 A
// and B, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t mma_idesc_f16_f32(int M, int N) {
    return (1u << 4)                          // D format: f32
           | (0u << 7) | (0u << 10)           // A, B format: f16
           | (0u << 15) | (0u << 16)          // A, B K-major
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// ----- programmatic dependent launch ---------------------------------------
// Wait until the grids this one depends on have completed and their writes are
// visible (a no-op when the launch had no programmatic dependency).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the dependent grid be scheduled before this one completes.
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----- tcgen05, one CTA (cta_group::1) --------------------------------------
__device__ __forceinline__ void tmem_alloc_1(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_1() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_1(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T with A (M x 16) and B (N x 16), both K-major in shared memory.
__device__ __forceinline__ void mma_f16_ss_1(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D (+)= A * B^T with A (M x 16) in tensor memory and B (N x 16) K-major in shared memory.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit_1(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns from registers (thread i writes
// lane quadrant base + i); tmem_wait_st waits until this thread's stores are done.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 32 lanes x 16 consecutive fp32 columns into registers (load and wait in one statement).
__device__ __forceinline__ void tmem_ld_32x32b_x16_sync(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Instruction descriptor of tcgen05.mma.kind::f16 with bf16 A and B, fp32
// accumulator, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t mma_idesc_bf16_f32(int M, int N) {
    return (1u << 4)                          // D format: f32
           | (1u << 7) | (1u << 10)           // A, B format: bf16
           | (0u << 15) | (0u << 16)          // A, B K-major
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace awq
