// common.cuh -- device helpers shared by the GEAR kernels (sm_100a only).
//
// Thin inline-PTX wrappers for the Blackwell features the kernels use:
// mbarriers, TMA tile loads (no multicast), tcgen05 tensor-memory allocation,
// MMA, commit and loads, plus the device error word that bounded waits set
// instead of trapping.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/gear.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "the GEAR kernels target sm_100a only"
#endif

namespace gear {

// ---------------------------------------------------------------- error word
// Kernels never trap. A bounded wait that gives up, or a debug check that
// fails, records a GEAR_ERR_* value here; gear_get_device_status() reads it.
extern __device__ int32_t g_device_status;

__device__ __forceinline__ void set_device_error(int32_t code) {
  atomicCAS(&g_device_status, 0, code);
}

// Bound of every spin on an mbarrier: 2 seconds of wall time (global timer),
// checked every 64 probes, plus an absolute cap on the number of probes.
constexpr uint64_t kSpinNanos = 2000000000ull;

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point
// (null if the driver does not provide it).
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
PFN_encodeTiled tensor_map_encoder();

// 2-D tensor map over a cache array of rows of `inner` 4-byte elements, boxes
// of `box_rows` whole rows; rows of 32, 64 or 128 bytes get the matching
// 16-byte-chunk swizzle (byte o of box row t at t*R + (o ^ (sw(t) << 4)),
// sw(t) = ((t*R) >> 7) & (R/16 - 1)), others none. Out-of-range rows read 0.
static inline bool cache_row_map(PFN_encodeTiled enc, CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                                 int inner, uint64_t rows, int box_rows) {
  const int row_bytes = inner * 4;
  const CUtensorMapSwizzle sw = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                  : CU_TENSOR_MAP_SWIZZLE_NONE;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)inner, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Codes as floats without integer conversion. Byte b of a code word is moved
// to mantissa bits 15..22 by one shift; each code of the byte is then masked
// into 1.0f: f = 1 + code * 2^(pos*BITS - 8), pos = index of the code inside
// its byte. The power of two 2^(8 - pos*BITS) is folded into a pre-scaled copy
// of q (keys) or applied once per channel at the end (values), both exact.
template <int BITS>
struct CodeFloats {
  static constexpr int kPerByte = 8 / BITS;
  static constexpr int kPerWord = 32 / BITS;
  // all codes of one 32-bit word, in channel order. `one` holds the bits of
  // 1.0f in a register, so that mask and exponent go into one LOP3 each.
  __device__ static __forceinline__ void word(uint32_t w, float (&f)[kPerWord], uint32_t one) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int sh = 15 - 8 * b;
      const uint32_t v = sh >= 0 ? (w << sh) : (w >> (-sh));
#pragma unroll
      for (int q = 0; q < kPerByte; ++q) {
        const uint32_t m = ((1u << BITS) - 1u) << (15 + q * BITS);
        f[b * kPerByte + q] = __uint_as_float((v & m) | one);
      }
    }
  }
  // weight that turns (f - 1) back into the code, for the code at channel c
  __host__ __device__ static constexpr float inv_weight(int c) {
    return (float)(1 << (8 - (c % kPerByte) * BITS));
  }
  // its inverse 2^(pos*BITS - 8), exactly (a power of two built from its bits)
  __device__ static __forceinline__ float weight(int c) {
    return __int_as_float((127 + (c % kPerByte) * BITS - 8) << 23);
  }
};

// Bytes of G groups' (scale, zero) pairs: fp32 pairs, or binary16 pairs.
__host__ __device__ constexpr int meta_row_bytes(int G, int meta_f16) { return G * (meta_f16 ? 4 : 8); }

// Token-group slots of a cache with per-channel key groups of g tokens: block
// 0 may end in a shorter group, every flushed block holds whole groups.
__host__ __device__ constexpr int channel_group_slots(int n_max, int g) { return (n_max + g - 1) / g + 1; }

// Row length of the stored Rf factors: r_max rounded up to a multiple of 4, so
// that one channel's row is a whole number of 16-byte vectors.
__host__ __device__ constexpr int rpad_of(int r_max) { return (r_max + 3) & ~3; }
constexpr uint32_t kSpinLimit = 1u << 26;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Next 1024-byte boundary of the shared window at or after p. The offset is
// added to p itself, so the result stays a shared-memory pointer to the
// compiler (shared loads and stores rather than generic ones).
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps (issuing nothing) until
// the phase completes or about `ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, sleeping between
// probes. Returns false (and records GEAR_ERR_TIMEOUT) if the barrier does not
// complete within `limit_ns` of wall time.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  const uint32_t every = limit_ns < kSpinNanos ? 1u : 64u;   // short bounds: check the clock each probe
  for (uint32_t i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if ((i % every) == 0 && global_timer_ns() - t0 > limit_ns) break;
  }
  set_device_error(GEAR_ERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kSpinNanos);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16/f16 inputs, f32 accumulate).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on the mbarrier once every previously issued tcgen05.mma of this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives row
// (warp's lane quarter + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// 32 lanes x 8 consecutive 32-bit columns (thread i: row quarter*32 + i).
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns (thread i: row quarter*32 + i).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for tcgen05.mma: 128-byte swizzled canonical
// layout. Fields: start address >> 4 (bits 0-13), leading-dimension byte offset
// >> 4 (16-29), stride-dimension byte offset >> 4 (32-45), descriptor version 1
// (bits 46-47), base offset 0, layout type 2 = 128B swizzle (bits 61-63).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16 with f32 accumulation.
//   c_format bits 4-5 = 1 (f32); a_format bits 7-9, b_format bits 10-12:
//   0 = f16, 1 = bf16; a_major bit 15, b_major bit 16 (1 = MN-major);
//   N >> 3 in bits 17-22; M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool bf16, bool a_mn, bool b_mn) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- launch set-up
// cudaFuncSetAttribute acts on the CURRENT device only, so a kernel's dynamic
// shared-memory limit has to be raised once on every device that launches it.
// Each launch site keeps one slot per device (devices 0 .. kMaxDevices-1)
// holding the largest size already set there. Host threads may race to set the
// same attribute, which is harmless; the slots are atomics so that the race is
// well defined. Devices beyond the table are set on every launch.
constexpr int kMaxDevices = 64;

template <typename Kern>
inline cudaError_t ensure_smem_limit(Kern kern, int bytes, std::atomic<int> (&slots)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && slots[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (cached) {
    int cur = slots[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !slots[dev].compare_exchange_weak(cur, bytes, std::memory_order_release)) {
    }
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

template <typename T>
struct dtype_of;
template <>
struct dtype_of<__half> { static constexpr int value = GEAR_F16; };
template <>
struct dtype_of<__nv_bfloat16> { static constexpr int value = GEAR_BF16; };
template <>
struct dtype_of<float> { static constexpr int value = GEAR_F32; };

}  // namespace gear
