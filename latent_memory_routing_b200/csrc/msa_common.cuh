// Shared device/host helpers of libmsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

// ---------------------------------------------------------------- host side

// Records `e` as the calling thread's last CUDA error; returns MSA_ERR_CUDA
// if e != cudaSuccess, MSA_OK otherwise.
int note_cuda(cudaError_t e);

// Launch-error check after a <<<>>> launch.
inline int check_launch() { return note_cuda(cudaGetLastError()); }

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms();  // SM count of the current device (cached per device)

// Sets a kernel's dynamic shared-memory limit once per (kernel, device), so
// that later calls -- including calls made while a stream is being captured
// into a CUDA graph -- only launch.
int ensure_smem_attr(const void* func, int bytes);

// ------------------------------------------ programmatic dependent launch
//
// The kernels of a step are launched as programmatic dependents of the work
// before them in the stream: a grid may be scheduled as soon as every CTA of
// the kernel before it has signalled (pdl_trigger) or exited, which overlaps
// the launch latency with that kernel's tail.  Ordering is unchanged: a
// kernel launched this way calls pdl_wait() before it reads or writes global
// memory, which waits for the previous grid's completion and the visibility
// of its writes (and that grid, if it was launched the same way, had itself
// waited for its predecessor).  Both are no-ops for a kernel launched
// without the dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note_cuda(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
}

// ---------------------------------------------------------- device status

// Device address of the current device's status word (first
// device-detected error since the last reset, 0 = none).  The word is a
// file-scope __device__ variable of api.cu; its address is looked up once per
// device and passed to kernels as a plain pointer.
int* device_status_ptr();

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------- debug build
//
// Built with -DMSA_DEBUG (libmsa_debug.so), every entry point checks the
// device-side index arrays it is given before any kernel reads through them,
// and waits for its own work.  A check launches a small validation kernel,
// waits for it and returns the device status word's error, if one is set
// (the word is not cleared), so a bad input comes back as an error status
// from the call that received it and the hot kernels never run on it.
// While the stream is being captured into a CUDA graph nothing waits: the
// validation kernels are captured too and record into the status word.  In
// the release build these functions are empty and compile away.
#ifdef MSA_DEBUG
// CSR offsets [n+1]: 0 <= off[0] <= off[1] <= ... <= off[n] <= total.
int debug_check_offsets(const int64_t* off, int n, int64_t total, cudaStream_t s);
// Per-query memory lengths [B]: 0 <= mem_len[b] <= m_cap.
int debug_check_mem_len(const int32_t* mem_len, int B, int m_cap, cudaStream_t s);
// End of an entry point: rc if it is an error; otherwise waits for the
// stream and returns a CUDA error or the status word's error, if any.
int debug_finish(int rc, cudaStream_t s);
#else
inline int debug_check_offsets(const int64_t*, int, int64_t, cudaStream_t) { return MSA_OK; }
inline int debug_check_mem_len(const int32_t*, int, int, cudaStream_t) { return MSA_OK; }
inline int debug_finish(int rc, cudaStream_t) { return rc; }
#endif

// ------------------------------------------------------------ element types

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) {
    return __bfloat162float(x);
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) {
    return __float2bfloat16_rn(x);
  }
};

// 16-byte vector <-> VEC floats (VEC = 4 for fp32, 8 for bf16).
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  static __device__ __forceinline__ uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                      __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint4 pack(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
// Streaming load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st16(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}

// ------------------------------------------------------------------- RoPE

// Inverse frequency base^(-2i/D) in double.
__device__ __forceinline__ double rope_inv_freq(double base, int i, int D) {
  return pow(base, -2.0 * (double)i / (double)D);
}

// (cos, sin) of the angle p * w.  The angle and its reduction to [-pi, pi]
// are done in double (exact to ~1e-12 rad for p < 2^31), so only the final
// float conversion of the reduced angle (<= 1.2e-7 rad) and sincosf itself
// add error: ~2e-7 absolute, independent of p.
__device__ __forceinline__ float2 rope_cs(int64_t p, double w) {
  const double two_pi = 6.283185307179586;  // 2*pi rounded to double
  double th = (double)p * w;
  double n = rint(th * (1.0 / two_pi));
  float r = (float)fma(-n, two_pi, th);
  float s, c;
  sincosf(r, &s, &c);
  return make_float2(c, s);
}

// -------------------------------------------------------------- searching

// Warp-cooperative search over a non-decreasing int64 array off[0..n]
// (off[0] = 0 <= x < off[n]): returns the largest d in [0, n) with
// off[d] <= x.  All 32 lanes must call it with the same arguments.
__device__ __forceinline__ int64_t warp_find_segment(const int64_t* off,
                                                     int64_t n, int64_t x) {
  const int lane = threadIdx.x & 31;
  int64_t lo = 0, hi = n;  // invariant: off[lo] <= x, answer in [lo, hi)
  while (hi - lo > 1) {
    const int64_t span = hi - lo;
    const int64_t step = (span + 31) / 32;
    const int64_t p = lo + (int64_t)lane * step;
    const bool ok = (p < hi) && (__ldg(off + p) <= x);
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    const int last = 31 - __clz(m);  // lane 0 always satisfies off[lo] <= x
    lo = lo + (int64_t)last * step;
    const int64_t nh = lo + step;
    hi = nh < hi ? nh : hi;
  }
  return lo;
}

// Order-preserving float <-> uint32 map: a < b  <=>  f2o(a) < f2o(b)
// (NaN maps above +inf for positive-sign NaN; callers filter NaN first).
__device__ __forceinline__ uint32_t f2o(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float o2f(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

}  // namespace msa
