// Device helpers shared by the BitLinear kernels (sm_100a only).
//
// Arithmetic that decides an integer code uses the explicit round-to-nearest
// intrinsics (__fmul_rn, __fadd_rn, __fdiv_rn, __fsqrt_rn) so that no
// multiply-add contraction can change a rounding, whatever the compiler flags.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <map>
#include <utility>

#define BN_DEV __device__ __forceinline__

namespace bitnet {

// ---------------------------------------------------------------------------
// error flag: set by a bounded wait that gave up; read by bitnet_device_error()
// ---------------------------------------------------------------------------
extern __device__ int g_device_error;

enum DeviceError : int {
  DEV_ERR_NONE = 0,
  DEV_ERR_TIMEOUT_FULL = 1,
  DEV_ERR_TIMEOUT_EMPTY = 2,
  DEV_ERR_TIMEOUT_A = 3,
  DEV_ERR_TIMEOUT_ACC = 4,
  DEV_ERR_TIMEOUT_CLUSTER = 5,
};

// ---------------------------------------------------------------------------
// A group of ternary weight matrices that share one activation tensor (the
// Q/K/V projections of an attention block, the up/gate projections of a gated
// FFN), computed by one launch.  A single product is a group of one.  CTAs (or
// output tiles) first[g] .. first[g+1]-1 of the grid work on matrix g.
// ---------------------------------------------------------------------------
constexpr int GROUP_MAX = 4;

struct LinGroup {
  const uint8_t* pkW[GROUP_MAX];
  const float* s_w[GROUP_MAX];
  void* Y[GROUP_MAX];
  int32_t* acc_dbg[GROUP_MAX];
  int N[GROUP_MAX];
  int first[GROUP_MAX + 1];
  int count;
};

// Index of the matrix that block b works on (uniform across the CTA).
BN_DEV int group_of(const LinGroup& g, int b) {
  int gi = 0;
#pragma unroll
  for (int j = 1; j < GROUP_MAX; ++j) gi += (j < g.count && b >= g.first[j]) ? 1 : 0;
  return gi;
}

// ---------------------------------------------------------------------------
// bf16 / vector helpers
// ---------------------------------------------------------------------------
BN_DEV float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
BN_DEV float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Read-only data of the whole call (weights, gamma): non-coherent path.
BN_DEV uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
BN_DEV float ldg_nc_f32(const float* p) {
  float r;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(p));
  return r;
}

// Data written by the previous kernel in the stream (activations, s_x),
// read after the programmatic-launch wait: plain coherent loads.  The asm is
// volatile so that the loads are issued where they are written (all at once,
// ahead of their first use) instead of being moved down to it.
BN_DEV uint4 ldg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
BN_DEV uint2 ldg_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
BN_DEV float ldg_f32(const float* p) {
  float r;
  asm volatile("ld.global.f32 %0, [%1];" : "=f"(r) : "l"(p));
  return r;
}

// Squared-ReLU gated unit, fp32 round-to-nearest: (r * r) * u, r = max(g, 0).
BN_DEV float relu2_times(float g, float u) {
  const float r = fmaxf(g, 0.0f);
  return __fmul_rn(__fmul_rn(r, r), u);
}

BN_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// p advanced to the next multiple of `align` (a power of two) bytes of the
// shared window, by pointer arithmetic on the shared array itself: the
// compiler then still knows that the result addresses shared memory (a round
// trip through an integer would make every access through it a generic one).
template <typename T>
BN_DEV T* smem_align(T* p, uint32_t align) {
  const uint32_t pad = (align - (smem_u32(p) & (align - 1u))) & (align - 1u);
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(p) + pad);
}

BN_DEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

BN_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
BN_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

BN_DEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

BN_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\t"
               "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}"
               :: "r"(smem_u32(bar)) : "memory");
}

BN_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\t"
               "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

BN_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after about
// two seconds of wall time, records `code` in g_device_error and returns false.
// With bail = true it also returns false as soon as another wait has given up;
// teardown waits (in-flight copies, MMAs) pass bail = false.
BN_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int code, bool bail = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (bail && *((volatile int*)&g_device_error) != 0) return false;
      if (globaltimer() - t0 > 2000000000ull) {
        atomicCAS(&g_device_error, 0, code);
        return false;
      }
    }
  }
  return true;
}

// Non-blocking test of a phase (never suspends the thread).
BN_DEV bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Cluster-scope acquire variant: pairs with remote arrives that release at
// cluster scope (writes into this CTA's shared memory by other CTAs).
BN_DEV bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

BN_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int code) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_try_wait_cluster(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (*((volatile int*)&g_device_error) != 0) return false;
      if (globaltimer() - t0 > 2000000000ull) {
        atomicCAS(&g_device_error, 0, code);
        return false;
      }
    }
  }
  return true;
}

// Warp-uniform variant for warps that go on to issue .sync.aligned tcgen05 ops.
BN_DEV bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int code) {
  const bool ok = mbar_wait(bar, parity, code);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// thread-block clusters: distributed shared memory, cluster barrier
// ---------------------------------------------------------------------------
BN_DEV uint32_t cluster_map(uint32_t local_smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem_addr), "r"(rank));
  return r;
}
BN_DEV void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}
BN_DEV void mbar_arrive_remote(uint32_t cluster_bar_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
               :: "r"(cluster_bar_addr) : "memory");
}
BN_DEV void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
BN_DEV void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory into
// another CTA's shared memory; completion is signalled on that CTA's mbarrier.
BN_DEV void bulk_copy_to_cluster(uint32_t dst_cluster_addr, const void* src, uint32_t bytes,
                                 uint32_t bar_cluster_addr) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst_cluster_addr), "r"(smem_u32(src)), "r"(bytes), "r"(bar_cluster_addr) : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until the source reads of this thread's committed bulk copies are done.
BN_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
BN_DEV void cp_async_16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst_smem), "l"(src), "r"(src_bytes) : "memory");
}
BN_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
BN_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

BN_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------
// Lets the next kernel in the stream be scheduled once every CTA of this grid
// has started (it still waits for this grid's results where it reads them).
BN_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Blocks until the grids this one depends on have completed and their writes
// are visible; returns at once when there are none.
BN_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// TMA (plain per-CTA loads and stores)
// ---------------------------------------------------------------------------
BN_DEV void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

BN_DEV void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :: "r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

BN_DEV void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// TMA bulk tensor store of a shared-memory box (out-of-bounds parts are dropped).
BN_DEV void tma_store_2d(const void* tmap, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               :: "l"(tmap), "r"(smem_u32(smem_src)), "r"(x), "r"(y) : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until this thread's committed bulk stores have completed their writes.
BN_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

BN_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, tensor memory)
// ---------------------------------------------------------------------------
BN_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
BN_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
BN_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               :: "r"(taddr), "r"(ncols) : "memory");
}
BN_DEV void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
BN_DEV void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] x B[smem desc]; kind::i8, int32 accumulate, cta_group::1.
BN_DEV void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                      uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
               :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
               : "memory");
}

// Arrive on an mbarrier of this CTA once every prior tcgen05 op of the thread is done.
BN_DEV void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

BN_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
BN_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Each lane of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
BN_DEV void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr),
         "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
         "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
         "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
         "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Each lane writes 16 consecutive 32-bit columns of its own TMEM lane.
BN_DEV void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :: "r"(taddr),
         "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
         "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Each lane reads 8 consecutive 32-bit columns of its own TMEM lane.
BN_DEV void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
      : "r"(taddr) : "memory");
}

// Each lane reads 16 consecutive 32-bit columns of its own TMEM lane.
BN_DEV void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
BN_DEV uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
  d |= (uint64_t)1u << 16;                          // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset
  d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                          // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::i8, s8 x s8 -> s32, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                              // D format s32
       | (1u << 7) | (1u << 10)                 // A, B signed 8-bit
       | ((uint32_t)(N >> 3) << 17)
       | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// host: launch with programmatic stream serialisation (and a cluster shape)
// ---------------------------------------------------------------------------
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, dim3 cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  unsigned n = 0;
  attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster.x * cluster.y * cluster.z > 1) {
    attrs[n].id = cudaLaunchAttributeClusterDimension;
    attrs[n].val.clusterDim.x = cluster.x;
    attrs[n].val.clusterDim.y = cluster.y;
    attrs[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// host: raise a kernel's dynamic shared-memory limit once per (kernel, device)
// ---------------------------------------------------------------------------
inline cudaError_t ensure_smem_limit(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> limit;   // largest limit set so far
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = limit.find({kernel, dev});
  if (it != limit.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) limit[{kernel, dev}] = bytes;
  return e;
}

}  // namespace bitnet
