// Host side of libinfini_attn: the C ABI declared in include/infini_attn.h.
//
// A forward runs, on the caller's stream:
//   linear rule (Eq. 8): update partials for every (b, h, segment, group) in
//     one launch, then one state launch that scans the segments in order,
//     writing the snapshots (M_{s-1}, z_{s-1}) and the final (M_S, z_S);
//   delta rule (Eq. 9), tensor cores: one update launch per segment, which
//     snapshots (M_{s-1}, z_{s-1}), computes the segment's partials and
//     reduces them into M, z inside each head's thread-block cluster;
//   delta rule, CUDA cores: a snapshot launch of (M_0, z_0), then per segment
//     one update launch (reads M_{s-1}) and one state launch (adds the
//     partials and snapshots M_s);
//   then one attention launch (Eq. 6, 7, 10) over every (b, h, segment,
//     query tile), reading the snapshots.
// The order "read with M_{s-1}, then update" of the pages holds because the
// attention kernel reads the snapshot of M_{s-1}, never the running state.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdio>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/infini_attn.h"
#include "common.cuh"
#include "simt.cuh"
#include "bwd_simt.cuh"
#include "bwd_mem.cuh"
#include "decode.cuh"
#include "rope.cuh"
#include "sm100_attn.cuh"
#include "sm100_update.cuh"
#include "sm100_delta.cuh"
#include "sm100_gemm.cuh"
#include "sm100_bwd.cuh"
#include "sm100_bwdmem.cuh"

namespace infini {
namespace {

constexpr int kChunk = 128;        // tokens per update chunk
constexpr int kSms = 148;          // B200 SM count: grid sizing (device independent, so plans are too)
constexpr int kTargetCtas = 4 * kSms;  // CUDA-core update grid size aim
constexpr size_t kAlign = 256;
// Internal flag of forward_impl (not in the header): run the memory update
// only -- no attention launch, no output -- for the decode step's fold.
constexpr int kFlagUpdateOnly = 0x1000;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ------------------------------------------------------------ launch accounting
enum Phase { kPhaseUpdate = 0, kPhaseState = 1, kPhaseAttn = 2, kPhasePre = 3, kPhaseProj = 4, kPhaseBwd = 5, kPhaseBwdTc = 6,
             kPhaseBwdMemTc = 7, kPhases = 8 };
std::atomic<long long> g_launches{0};
std::atomic<int> g_profile_mask{0};
struct EventPair {
  int phase;
  cudaEvent_t a, b;
  unsigned long long ctx;  // the context the events belong to
};
std::mutex g_prof_mu;
std::vector<EventPair> g_prof;
// Timing events already read out, for reuse (an event belongs to the context
// it was created in): creating two events per timed launch would add host time
// to every timed call.
std::vector<std::pair<unsigned long long, cudaEvent_t>> g_event_pool;
unsigned long long current_context_id();

cudaEvent_t take_timing_event(unsigned long long ctx) {
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (size_t i = 0; i < g_event_pool.size(); ++i)
      if (g_event_pool[i].first == ctx) {
        cudaEvent_t e = g_event_pool[i].second;
        g_event_pool[i] = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
      }
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// Counts one kernel launch and, when its phase is being timed, brackets it
// with events on `stream`.  Construct right before the launch, destroy
// right after it.
struct LaunchScope {
  int phase;
  cudaStream_t stream;
  cudaEvent_t a = nullptr, b = nullptr;
  unsigned long long ctx = 0;
  LaunchScope(int ph, cudaStream_t st) : phase(ph), stream(st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_profile_mask.load(std::memory_order_relaxed) & (1 << ph)) {
      ctx = current_context_id();
      a = take_timing_event(ctx);
      b = a ? take_timing_event(ctx) : nullptr;
      if (a && b) {
        cudaEventRecord(a, stream);
      } else {
        if (a) cudaEventDestroy(a);
        a = b = nullptr;
      }
    }
  }
  ~LaunchScope() {
    if (a && b) {
      cudaEventRecord(b, stream);
      std::lock_guard<std::mutex> lk(g_prof_mu);
      g_prof.push_back({phase, a, b, ctx});
    }
  }
};

struct Plan {
  int B, H, N, dk, dv, mode, S, G, cpb, nseg_part;
  long long L;
  bool delta, f32, tc;
  size_t off_snapM, off_snapz, off_part, off_ctr, total;
};

// Workspace: per-segment snapshots of M_{s-1} (bf16 [dk][dv] for the tensor
// cores, fp32 otherwise) and z_{s-1} (fp32), and the update partials
// ([BH][S][G] for the linear scan, [BH][1][G] reused per segment for delta).
int make_plan(int B, int H, long long L, int N, int dk, int dv, int mode, int flags, Plan* p) {
  if (B <= 0 || H <= 0 || L <= 0 || N <= 0 || dk <= 0 || dv <= 0) return INFINI_ERR_INVALID_ARG;
  if ((mode & ~(INFINI_DELTA | INFINI_F32)) != 0) return INFINI_ERR_UNSUPPORTED;
  if (dk > 128 || dv > 128) return INFINI_ERR_UNSUPPORTED;
  p->B = B; p->H = H; p->L = L; p->N = N; p->dk = dk; p->dv = dv; p->mode = mode;
  p->delta = (mode & INFINI_DELTA) != 0;
  p->f32 = (mode & INFINI_F32) != 0;
  p->tc = !p->f32 && dk == 128 && dv == 128 && !(flags & INFINI_FLAG_FORCE_SIMT);
  const long long S = (L + N - 1) / N;
  const long long BH = (long long)B * H;
  if (S > (1 << 30) || BH * S > (1LL << 31) / 4 || L > (1LL << 31) - 1) return INFINI_ERR_UNSUPPORTED;
  p->S = (int)S;
  const int chunks_per_seg = (std::min<long long>(N, L) + kChunk - 1) / kChunk;
  const long long units = p->delta ? BH : BH * S;  // CTAs per launch before grouping
  long long cpb;
  if (p->tc) {
    // Tensor cores: long CTAs (the chunk pipeline hides load latency), about one
    // wave; the delta rule's G CTAs of a head form one cluster of at most 8.
    long long G = std::max<long long>(1, kSms / units);
    G = std::min<long long>(G, p->delta ? tc::kMaxDeltaCluster : chunks_per_seg);
    G = std::min<long long>(G, chunks_per_seg);
    // One segment with its attention (a streaming step): the update runs
    // alongside the attention, which sets the call's length, so it takes about
    // an eighth of the SMs (two CTAs per head at 8 heads) and leaves the rest
    if (S == 1 && !(flags & kFlagUpdateOnly))
      G = std::max<long long>(1, std::min<long long>(G, (kSms / 8) / units));
    cpb = (chunks_per_seg + G - 1) / G;
  } else {
    cpb = (units * chunks_per_seg + kTargetCtas - 1) / kTargetCtas;
    cpb = std::max<long long>(1, std::min<long long>(cpb, chunks_per_seg));
  }
  p->cpb = (int)cpb;
  p->G = (int)((chunks_per_seg + cpb - 1) / cpb);
  p->nseg_part = p->delta ? 1 : p->S;
  const size_t E = (size_t)dk * dv;
  size_t off = 0;
  p->off_snapM = off;
  off = align_up(off + (size_t)BH * S * E * (p->tc ? 2 : 4));
  p->off_snapz = off;
  off = align_up(off + (size_t)BH * S * dk * 4);
  p->off_part = off;
  off = align_up(off + (size_t)BH * p->nseg_part * p->G * (E + dk) * 4);
  p->off_ctr = off;  // work counter of the persistent attention kernel
  off = align_up(off + (p->tc ? 8 : 0));
  p->total = off;
  return INFINI_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Unique id of the CUDA context current on this thread (0 if none or on
// failure).  Per-context caches key on it rather than on the device ordinal:
// a context that is destroyed and recreated (cudaDeviceReset, a primary
// context reset) gets a new id, so nothing cached for the old one is reused.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// 4-D map over a [B, H, L, 128] bf16 tensor with element strides st[0..2]
// (d contiguous); box 64 x 128 tokens, 128-byte swizzle.
bool encode_bhld(CUtensorMap* m, const void* ptr, int B, int H, long long L, const long long st[3],
                 uint32_t box_rows = 128) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {128, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 2-D map over rows x 128 bf16 (row-major), box 64 x 128 rows, 128-byte swizzle.
bool encode_rows(CUtensorMap* m, const void* ptr, long long rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool ranges_overlap(const void* a, size_t an, const void* b, size_t bn) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + bn && y < x + an;
}
size_t extent_bytes(const long long st[3], int B, int H, long long L, int d, size_t es) {
  return (size_t)(((long long)(B - 1) * st[0] + (long long)(H - 1) * st[1] + (L - 1) * st[2] + d) * (long long)es);
}

int check_device(bool need_tc) {
  (void)need_tc;
  // the answer for a context does not change: asked once per context (and thread)
  thread_local unsigned long long ok_ctx = 0;
  const unsigned long long ctx = current_context_id();
  if (ctx != 0 && ctx == ok_ctx) return INFINI_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INFINI_ERR_DEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return INFINI_ERR_DEVICE;
  if (major != 10) return INFINI_ERR_DEVICE;
  ok_ctx = ctx;
  return INFINI_OK;
}

// The fork and join events of one-segment calls, created once per thread and
// context (a pair shared between threads could interleave their records).
bool fork_events(cudaEvent_t* ev_fork, cudaEvent_t* ev_join) {
  struct Pair {
    unsigned long long ctx;
    cudaEvent_t fork, join;
  };
  thread_local std::vector<Pair> pairs;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return false;
  for (const Pair& e : pairs)
    if (e.ctx == ctx) {
      *ev_fork = e.fork;
      *ev_join = e.join;
      return true;
    }
  Pair e{ctx, nullptr, nullptr};
  if (cudaEventCreateWithFlags(&e.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&e.join, cudaEventDisableTiming) != cudaSuccess) {
    if (e.fork) cudaEventDestroy(e.fork);
    cudaGetLastError();
    return false;
  }
  pairs.push_back(e);
  *ev_fork = e.fork;
  *ev_join = e.join;
  return true;
}

// The CUDA error behind the most recent INFINI_ERR_LAUNCH (any thread).
std::atomic<int> g_last_cuda_error{0};
int note_cuda_error(cudaError_t e) {
  g_last_cuda_error.store((int)e);
  return INFINI_ERR_LAUNCH;
}
int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? INFINI_OK : note_cuda_error(e);
}

// What the local attention (Eq. 6) reads: q, k themselves, or their rotated
// copies in the workspace when position embeddings are on (then qm is the
// un-rotated q that sigma(Q) of the memory read takes).
struct LocalQK {
  const void* q;
  const void* k;
  long long qs[3], ks[3];
  const void* qm;  // nullptr: no position embeddings
};

size_t rope_bytes(const infini_attn_params& p) {
  if (p.rope_base == 0.0) return 0;
  const size_t es = (p.mode & INFINI_F32) ? 4 : 2;
  return 2 * align_up((size_t)p.B * p.H * (size_t)p.L * p.dk * es);
}

// Rotated copies of q and k (contiguous [B, H, L, dk]) at `dst`.
int run_rope(const infini_attn_params& p, char* dst, LocalQK* loc) {
  const bool f32 = (p.mode & INFINI_F32) != 0;
  const size_t es = f32 ? 4 : 2;
  const size_t one = align_up((size_t)p.B * p.H * (size_t)p.L * p.dk * es);
  RopeArgs ra;
  memset(&ra, 0, sizeof(ra));
  ra.q = p.q; ra.k = p.k; ra.qr = dst; ra.kr = dst + one;
  for (int i = 0; i < 3; ++i) {
    ra.qs[i] = p.q_stride[i];
    ra.ks[i] = p.k_stride[i];
  }
  ra.L = p.L; ra.offset = p.rope_offset; ra.B = p.B; ra.H = p.H; ra.dk = p.dk;
  for (int i = 0; i < p.dk / 2; ++i) ra.inv_freq[i] = pow(p.rope_base, -2.0 * i / p.dk);
  // 16-byte vectors need dk % 8 == 0 and rows that start on 16 bytes
  bool vec = p.dk % 8 == 0 && reinterpret_cast<uintptr_t>(p.q) % 16 == 0 && reinterpret_cast<uintptr_t>(p.k) % 16 == 0;
  for (int i = 0; i < 3; ++i)
    vec = vec && (p.q_stride[i] * (long long)es) % 16 == 0 && (p.k_stride[i] * (long long)es) % 16 == 0;
  const int E = vec ? 8 : 2;
  // block: the dk / E element groups of rows_per tokens; grid: tokens x heads
  const int groups = p.dk / E;
  const int rows_per = std::max(1, 256 / groups);
  const long long bx = (p.L + rows_per - 1) / rows_per;
  if (bx >= (1LL << 31)) return INFINI_ERR_UNSUPPORTED;
  const dim3 block((unsigned)groups, (unsigned)rows_per);
  // up to 8 heads per thread: the sine/cosine of a token's pairs serve them all
  const dim3 grid((unsigned)bx, (unsigned)std::min<long long>(((long long)p.B * p.H + 7) / 8, 65535));
  {
    LaunchScope ls(kPhasePre, p.stream);
    if (f32) {
      if (vec) rope_kernel<float, 8><<<grid, block, 0, p.stream>>>(ra);
      else rope_kernel<float, 2><<<grid, block, 0, p.stream>>>(ra);
    } else {
      if (vec) rope_kernel<__nv_bfloat16, 8><<<grid, block, 0, p.stream>>>(ra);
      else rope_kernel<__nv_bfloat16, 2><<<grid, block, 0, p.stream>>>(ra);
    }
  }
  loc->q = ra.qr;
  loc->k = ra.kr;
  const long long st[3] = {(long long)p.H * p.L * p.dk, p.L * p.dk, p.dk};
  for (int i = 0; i < 3; ++i) loc->qs[i] = loc->ks[i] = st[i];
  loc->qm = p.q;
  return launch_status();
}

template <typename T>
int run_simt(const infini_attn_params& p, const Plan& pl, char* ws, float scale, const LocalQK& loc,
             float* adot = nullptr, float* lse = nullptr) {
  Geo g;
  g.B = p.B; g.H = p.H; g.L = p.L; g.N = p.N; g.dk = p.dk; g.dv = p.dv; g.S = pl.S;
  for (int i = 0; i < 3; ++i) {
    g.qs[i] = p.q_stride[i]; g.ks[i] = p.k_stride[i]; g.vs[i] = p.v_stride[i]; g.os[i] = p.o_stride[i];
  }
  float* snapM = reinterpret_cast<float*>(ws + pl.off_snapM);
  float* snapz = reinterpret_cast<float*>(ws + pl.off_snapz);
  float* part = reinterpret_cast<float*>(ws + pl.off_part);
  const int BH = p.B * p.H, E = p.dk * p.dv;
  const dim3 sgrid((E + p.dk + 255) / 256, BH);
  const size_t upd_smem = (size_t)(32 * p.dk + 32 * p.dv + 32 + E + p.dk) * 4;
  cudaFuncSetAttribute(simt_update_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)upd_smem);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  if (!pl.delta) {
    {
      LaunchScope ls(kPhaseUpdate, p.stream);
      simt_update_kernel<T><<<BH * pl.S * pl.G, 256, upd_smem, p.stream>>>(k, v, g, 0, pl.S, pl.G, pl.cpb, nullptr,
                                                                            nullptr, part);
    }
    {
      LaunchScope ls(kPhaseState, p.stream);
      state_kernel<<<sgrid, 256, 0, p.stream>>>(p.M, p.z, part, p.dk, p.dv, pl.S, 0, 0, pl.S, pl.G, snapM, nullptr,
                                                snapz, nullptr);
    }
  } else {
    {
      LaunchScope ls(kPhaseState, p.stream);
      state_kernel<<<sgrid, 256, 0, p.stream>>>(p.M, p.z, part, p.dk, p.dv, pl.S, 2, 0, 1, pl.G, snapM, nullptr,
                                                snapz, nullptr);
    }
    for (int s = 0; s < pl.S; ++s) {
      {
        LaunchScope ls(kPhaseUpdate, p.stream);
        simt_update_kernel<T><<<BH * pl.G, 256, upd_smem, p.stream>>>(k, v, g, s, 1, pl.G, pl.cpb, snapM, snapz,
                                                                       part);
      }
      LaunchScope ls(kPhaseState, p.stream);
      state_kernel<<<sgrid, 256, 0, p.stream>>>(p.M, p.z, part, p.dk, p.dv, pl.S, 1, s, 1, pl.G, snapM, nullptr,
                                                snapz, nullptr);
    }
  }
  if (p.flags & kFlagUpdateOnly) return launch_status();
  const int QT = (p.N + 31) / 32;
  const size_t attn_smem = (size_t)(32 * (p.dk + 1) + 32 * p.dv + 32 * p.dk) * 4;
  cudaFuncSetAttribute(simt_attn_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn_smem);
  Geo ga = g;  // the local attention's q, k (rotated copies under position embeddings)
  for (int i = 0; i < 3; ++i) {
    ga.qs[i] = loc.qs[i];
    ga.ks[i] = loc.ks[i];
    ga.qms[i] = p.q_stride[i];
  }
  LaunchScope ls(kPhaseAttn, p.stream);
  simt_attn_kernel<T><<<(unsigned)((long long)QT * BH * pl.S), 256, attn_smem, p.stream>>>(
      static_cast<const T*>(loc.q), static_cast<const T*>(loc.k), v, p.beta, static_cast<T*>(p.out), ga, scale, QT,
      snapM, snapz, static_cast<const T*>(loc.qm), adot, lse);
  return launch_status();
}

// A second stream of this library in the current context (non-blocking,
// created on first use), for work that may overlap the caller's stream.
cudaStream_t side_stream() {
  static std::mutex mu;
  static std::vector<std::pair<unsigned long long, cudaStream_t>> streams;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  for (const auto& e : streams)
    if (e.first == ctx) return e.second;
  cudaStream_t st = nullptr;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  streams.emplace_back(ctx, st);
  return st;
}

// Workspace the library allocates itself comes from a stream-ordered memory
// pool of its own, one per context, whose release threshold keeps freed
// blocks for the next call: repeated calls of one shape take nothing from the
// driver after the first (the device's default pool, with its threshold of 0,
// hands memory back at every synchronization, and mapping gigabytes again
// costs milliseconds).  infini_attn_trim_workspace() returns what is unused.
std::mutex g_pool_mu;
std::vector<std::pair<unsigned long long, cudaMemPool_t>> g_pools;

cudaMemPool_t workspace_pool() {
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  for (const auto& e : g_pools)
    if (e.first == ctx) return e.second;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  cudaMemPoolProps props;
  memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool = nullptr;
  if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  uint64_t keep = ~0ull;
  if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) cudaGetLastError();
  g_pools.emplace_back(ctx, pool);
  return pool;
}

// Stream-ordered workspace allocation (released with cudaFreeAsync).
bool ws_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
  cudaMemPool_t pool = workspace_pool();
  const cudaError_t e =
      pool != nullptr ? cudaMallocFromPoolAsync(ptr, bytes, pool, stream) : cudaMallocAsync(ptr, bytes, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return true;
}

// The dynamic shared-memory limit is an attribute of a function in the
// current context: set it for the tensor-core kernels once for every context
// the process uses (an unknown context id, 0, sets it on every call).
int set_tc_smem_limits() {
  static std::mutex mu;
  static std::vector<unsigned long long> done;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(mu);
  if (ctx != 0 && std::find(done.begin(), done.end(), ctx) != done.end()) return INFINI_OK;
  if (cudaFuncSetAttribute(tc::attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tc::kAttnSmem) != cudaSuccess ||
      cudaFuncSetAttribute(tc::attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tc::kAttnSmem) != cudaSuccess ||
      cudaFuncSetAttribute(tc::mem_update_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tc::UpdSmem::BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(tc::delta_update_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tc::DeltaSmem::BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(tc::gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kGemmSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc::bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kDQSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc::bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kKVSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc::bwd_qmem_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kQmSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc::bwd_upd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kUpSmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(tc::bwd_outer_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kOtSmem) !=
          cudaSuccess)
    return INFINI_ERR_LAUNCH;
  if (ctx != 0) done.push_back(ctx);
  return INFINI_OK;
}

// 2-D map over a row-major bf16 matrix [rows, cols] with a row stride of ld
// elements; box box_c x box_r, 128-byte swizzle (box_c = 64).
bool encode_mat(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld, uint32_t box_c,
                uint32_t box_r) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {box_c, box_r};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// C[M, N] = A[M, K] B[K, N], row-major bf16 with row strides lda, ldb, ldc
// (elements), fp32 accumulation: the tcgen05 GEMM.  Needs N, K, lda, ldb, ldc
// multiples of 8 and 16-byte aligned bases (TMA rows start on 16 bytes).
int gemm_tc(const void* A, long long lda, const void* Bm, long long ldb, void* C, long long ldc, long long M, long long N,
            long long K, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) return INFINI_ERR_INVALID_ARG;
  if (N % 8 || K % 8 || lda % 8 || ldb % 8 || ldc % 8 || lda < K || ldb < N || ldc < N) return INFINI_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(A) % 16 || reinterpret_cast<uintptr_t>(Bm) % 16 || reinterpret_cast<uintptr_t>(C) % 16)
    return INFINI_ERR_UNSUPPORTED;
  if (M >= (1LL << 31) || N >= (1LL << 31) || K >= (1LL << 31)) return INFINI_ERR_UNSUPPORTED;
  const long long tiles_m = (M + tc::kGemmBM - 1) / tc::kGemmBM, tiles_n = (N + tc::kGemmBN - 1) / tc::kGemmBN;
  if (tiles_m * tiles_n >= (1LL << 31)) return INFINI_ERR_UNSUPPORTED;
  if (!get_encode()) return INFINI_ERR_DEVICE;
  CUtensorMap tm_a, tm_b;
  if (!encode_mat(&tm_a, A, M, K, lda, 64, tc::kGemmBM) || !encode_mat(&tm_b, Bm, K, N, ldb, 64, tc::kGemmBK))
    return INFINI_ERR_LAUNCH;
  if (set_tc_smem_limits() != INFINI_OK) return INFINI_ERR_LAUNCH;
  tc::GemmArgs ga;
  ga.C = static_cast<__nv_bfloat16*>(C);
  ga.ldc = ldc;
  ga.M = (int)M;
  ga.N = (int)N;
  ga.K = (int)K;
  ga.tiles_m = (int)tiles_m;
  ga.tiles_n = (int)tiles_n;
  int dev = 0, sms = kSms;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = kSms;
  LaunchScope ls(kPhaseProj, st);
  tc::gemm_tc_kernel<<<(unsigned)std::min<long long>(tiles_m * tiles_n, sms), tc::kGemmThreads, tc::kGemmSmem, st>>>(
      tm_a, tm_b, ga);
  return launch_status();
}

// Extra outputs of a forward run for the backward's recomputation.
struct FwdExtra {
  float* snapM32;       // fp32 [BH][S][dk][dv] snapshots of M^(s)
  float* adot;          // [B*H*L][128] A_dot
  float* lse2;          // [B*H*L] row log2-sum-exp2 of the scaled scores
};

int run_tc(const infini_attn_params& p, const Plan& pl, char* ws, float scale, const LocalQK& loc,
           const FwdExtra* extra = nullptr) {
  // tm_k: the keys of the memory update (un-rotated); tm_qa / tm_ka: the
  // local attention's queries and keys
  CUtensorMap tm_qa, tm_k, tm_ka, tm_v, tm_mt;
  __nv_bfloat16* snapM16 = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_snapM);
  float* snapz = reinterpret_cast<float*>(ws + pl.off_snapz);
  float* part = reinterpret_cast<float*>(ws + pl.off_part);
  const int BH = p.B * p.H, E = 128 * 128;
  if (!encode_bhld(&tm_qa, loc.q, p.B, p.H, p.L, loc.qs) || !encode_bhld(&tm_k, p.k, p.B, p.H, p.L, p.k_stride) ||
      !encode_bhld(&tm_ka, loc.k, p.B, p.H, p.L, loc.ks) || !encode_bhld(&tm_v, p.v, p.B, p.H, p.L, p.v_stride) ||
      !encode_rows(&tm_mt, snapM16, (long long)BH * pl.S * 128))
    return INFINI_ERR_LAUNCH;
  if (set_tc_smem_limits() != INFINI_OK) return INFINI_ERR_LAUNCH;
  const dim3 sgrid((E + 128 + 255) / 256, BH);
  tc::UpdArgs ua;
  ua.partial = part; ua.M = p.M; ua.z = p.z; ua.snapM = snapM16; ua.snapzw = snapz;
  ua.snapM32 = extra ? extra->snapM32 : nullptr;
  ua.B = p.B; ua.H = p.H; ua.S = pl.S; ua.N = p.N; ua.L = p.L;
  ua.G = pl.G; ua.cpb = pl.cpb;
  // One segment (a streaming step): the attention reads only the snapshot of
  // (M_0, z_0), which the update never writes after its start, so once the
  // snapshot is taken the update runs on a second stream and the attention
  // follows the snapshot on the caller's stream, as a programmatic dependent
  // (its setup overlaps the snapshot kernel; it reads nothing before the
  // snapshot is complete); the caller's stream then waits for the update
  // (event fork and join).  The snapshot kernel also zeroes the attention's
  // work counter.
  unsigned int* ctr = reinterpret_cast<unsigned int*>(ws + pl.off_ctr);
  cudaStream_t us = p.stream;  // the update's stream
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  const bool fork = pl.S == 1 && !(p.flags & kFlagUpdateOnly) && extra == nullptr;
  // Otherwise the attention's work counter is zeroed before the update, so
  // that the attention launch directly follows the update's last kernel (a
  // programmatic dependent of it, like the streaming case's).
  if (!fork && !(p.flags & kFlagUpdateOnly) && cudaMemsetAsync(ctr, 0, sizeof(unsigned int), p.stream) != cudaSuccess)
    return note_cuda_error(cudaGetLastError());
  if (fork) {
    {
      LaunchScope ls(kPhaseState, p.stream);
      state_kernel<<<sgrid, 256, 0, p.stream>>>(p.M, p.z, part, 128, 128, 1, 2, 0, 1, pl.G, nullptr, snapM16, snapz, ctr);
    }
    cudaStream_t side = side_stream();
    if (side != nullptr && fork_events(&ev_fork, &ev_join) && cudaEventRecord(ev_fork, p.stream) == cudaSuccess &&
        cudaStreamWaitEvent(side, ev_fork, 0) == cudaSuccess) {
      us = side;
    } else {
      cudaGetLastError();
    }
    ua.snapM = nullptr;  // taken above: the update kernels skip it
    ua.snapzw = nullptr;
  }
  // the caller's stream waits for the update's stream
  auto join = [&]() {
    if (ev_join != nullptr && us != p.stream) {
      if (cudaEventRecord(ev_join, us) != cudaSuccess || cudaStreamWaitEvent(p.stream, ev_join, 0) != cudaSuccess)
        cudaGetLastError();
    }
  };
  if (!pl.delta) {
    ua.seg0 = 0; ua.nseg = pl.S;
    {
      LaunchScope ls(kPhaseUpdate, us);
      tc::mem_update_tc_kernel<<<BH * pl.S * pl.G, tc::UpdWarps::THREADS, tc::UpdSmem::BYTES, us>>>(tm_k, tm_v, ua);
    }
    LaunchScope ls(kPhaseState, us);
    state_kernel<<<sgrid, 256, 0, us>>>(p.M, p.z, part, 128, 128, pl.S, 0, 0, pl.S, pl.G,
                                              extra ? extra->snapM32 : nullptr, fork ? nullptr : snapM16,
                                              fork ? nullptr : snapz, nullptr);
  } else {
    ua.nseg = 1;
    // 64-token chunks: K and V maps with 64-row boxes
    CUtensorMap tm_k64, tm_v64;
    if (!encode_bhld(&tm_k64, p.k, p.B, p.H, p.L, p.k_stride, tc::kDChunk) ||
        !encode_bhld(&tm_v64, p.v, p.B, p.H, p.L, p.v_stride, tc::kDChunk)) {
      join();
      return INFINI_ERR_LAUNCH;
    }
    // one cluster of G CTAs per head; G <= 8 (plan).  Segments after the
    // first launch as programmatic dependents of the previous segment's
    // update (their K, V loads start while it finishes; M, z wait for it).
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(BH * pl.G);
    cfg.blockDim = dim3(tc::kDeltaThreads);
    cfg.dynamicSmemBytes = tc::DeltaSmem::BYTES;
    cfg.stream = us;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    for (int s = 0; s < pl.S; ++s) {
      // snapshot of M_{s-1}, z_{s-1} for segment s, then the partials of
      // segment s, reduced inside each head's cluster into M, z
      ua.seg0 = s;
      cfg.numAttrs = s > 0 ? 2 : 1;
      LaunchScope ls(kPhaseUpdate, us);
      const cudaError_t e = cudaLaunchKernelEx(&cfg, tc::delta_update_tc_kernel, tm_k64, tm_v64, ua);
      if (e != cudaSuccess) {
        cudaGetLastError();
        join();
        return note_cuda_error(e);
      }
    }
  }
  if (p.flags & kFlagUpdateOnly) return launch_status();
  tc::AttnArgs aa;
  aa.beta = p.beta; aa.snapz = snapz; aa.out = static_cast<__nv_bfloat16*>(p.out);
  aa.B = p.B; aa.H = p.H; aa.S = pl.S; aa.T = (p.N + 127) / 128; aa.L = p.L; aa.N = p.N;
  aa.scale_log2 = scale * 1.4426950408889634f;
  for (int i = 0; i < 3; ++i) {
    aa.os[i] = p.o_stride[i];
    aa.qms[i] = p.q_stride[i];
  }
  aa.qm = static_cast<const __nv_bfloat16*>(loc.qm);
  aa.adot = extra ? extra->adot : nullptr;
  aa.lse2 = extra ? extra->lse2 : nullptr;
  // Scheduling groups of GS segments: about one wave of CTAs per group.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const long long NS = (long long)BH * pl.S;
  // Pairs of query tiles per CTA, unless that leaves SMs idle (short streaming steps):
  // then one query tile per CTA.
  // pairs of query tiles per item when they fill the GPU, else one tile per
  // item with its key tiles split between the two softmax warpgroups
  aa.single = NS * ((aa.T + 1) / 2) < sms ? 2 : 0;
  if (p.flags & INFINI_FLAG_ATTN_SINGLE) aa.single = 1;
  if (p.flags & INFINI_FLAG_ATTN_PAIRS) aa.single = 0;
  if (p.flags & INFINI_FLAG_ATTN_SPLIT) aa.single = 2;
  aa.P = aa.single ? aa.T : (aa.T + 1) / 2;
  aa.GS = (int)std::max<long long>(1, std::min<long long>(NS, (sms + aa.P - 1) / aa.P));
  const long long groups = (NS + aa.GS - 1) / aa.GS;
  // persistent: one CTA per SM, or one per work item when there are fewer
  const long long items = groups * aa.GS * aa.P;
  aa.work_counter = ctr;
  if (items >= (1LL << 31)) {
    join();
    return INFINI_ERR_UNSUPPORTED;
  }
  {
    LaunchScope ls(kPhaseAttn, p.stream);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)std::min<long long>(items, sms));
    cfg.blockDim = dim3(tc::kAttnThreads);
    cfg.dynamicSmemBytes = tc::kAttnSmem;
    cfg.stream = p.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;  // a programmatic dependent of the kernel before it (snapshot, scan or update)
    const cudaError_t e = aa.single == 2
                              ? cudaLaunchKernelEx(&cfg, tc::attn_tc_kernel<true>, tm_qa, tm_ka, tm_v, tm_mt, aa)
                              : cudaLaunchKernelEx(&cfg, tc::attn_tc_kernel<false>, tm_qa, tm_ka, tm_v, tm_mt, aa);
    if (e != cudaSuccess) {
      cudaGetLastError();
      join();
      return note_cuda_error(e);
    }
  }
  const int rc = launch_status();
  join();
  return rc;
}

bool tc_layout_ok(const infini_attn_params& p) {
  // the cluster reduction of the delta rule moves M and z in 16-byte vectors
  if (reinterpret_cast<uintptr_t>(p.M) % 16 != 0 || reinterpret_cast<uintptr_t>(p.z) % 16 != 0) return false;
  const void* ptrs[4] = {p.q, p.k, p.v, p.out};
  const long long* sts[4] = {p.q_stride, p.k_stride, p.v_stride, p.o_stride};
  for (int t = 0; t < 4; ++t) {
    if (reinterpret_cast<uintptr_t>(ptrs[t]) % 16 != 0) return false;
    for (int i = 0; i < 3; ++i)
      if (sts[t][i] <= 0 || (sts[t][i] * 2) % 16 != 0 || sts[t][i] * 2 >= (1LL << 40)) return false;
  }
  return true;
}

int forward_impl(infini_attn_params p) {
  const bool update_only = (p.flags & kFlagUpdateOnly) != 0;
  if (!p.q || !p.k || !p.v || !p.beta || !p.M || !p.z || (!p.out && !update_only)) return INFINI_ERR_INVALID_ARG;
  Plan pl;
  int rc = make_plan(p.B, p.H, p.L, p.N, p.dk, p.dv, p.mode, p.flags, &pl);
  if (rc != INFINI_OK) return rc;
  // default contiguous strides
  auto fill = [&](long long st[3], int d) {
    if (st[0] == 0 && st[1] == 0 && st[2] == 0) {
      st[2] = d;
      st[1] = p.L * d;
      st[0] = (long long)p.H * p.L * d;
    }
  };
  fill(p.q_stride, p.dk);
  fill(p.k_stride, p.dk);
  fill(p.v_stride, p.dv);
  fill(p.o_stride, p.dv);
  for (int i = 0; i < 3; ++i)
    if (p.q_stride[i] < 0 || p.k_stride[i] < 0 || p.v_stride[i] < 0 || p.o_stride[i] <= 0)
      return INFINI_ERR_INVALID_ARG;
  const size_t es = pl.f32 ? 4 : 2;
  const size_t out_ext = update_only ? 0 : extent_bytes(p.o_stride, p.B, p.H, p.L, p.dv, es);
  if (ranges_overlap(p.out, out_ext, p.q, extent_bytes(p.q_stride, p.B, p.H, p.L, p.dk, es)) ||
      ranges_overlap(p.out, out_ext, p.k, extent_bytes(p.k_stride, p.B, p.H, p.L, p.dk, es)) ||
      ranges_overlap(p.out, out_ext, p.v, extent_bytes(p.v_stride, p.B, p.H, p.L, p.dv, es)) ||
      ranges_overlap(p.out, out_ext, p.M, (size_t)p.B * p.H * p.dk * p.dv * 4) ||
      ranges_overlap(p.out, out_ext, p.z, (size_t)p.B * p.H * p.dk * 4) ||
      ranges_overlap(p.out, out_ext, p.beta, (size_t)p.H * 4) ||
      ranges_overlap(p.M, (size_t)p.B * p.H * p.dk * p.dv * 4, p.z, (size_t)p.B * p.H * p.dk * 4))
    return INFINI_ERR_INVALID_ARG;
  const bool rope = p.rope_base != 0.0;
  if (rope && !(p.rope_base > 0.0 && std::isfinite(p.rope_base))) return INFINI_ERR_INVALID_ARG;
  if (rope && p.dk % 2 != 0) return INFINI_ERR_UNSUPPORTED;
  if (pl.tc && !tc_layout_ok(p)) {
    // The tensor-core kernels need TMA-compatible strides; other layouts run on CUDA cores.
    rc = make_plan(p.B, p.H, p.L, p.N, p.dk, p.dv, p.mode, p.flags | INFINI_FLAG_FORCE_SIMT, &pl);
    if (rc != INFINI_OK) return rc;
  }
  // workspace: the plan's buffers, then the rotated q, k under position embeddings
  const size_t need = pl.total + rope_bytes(p);
  if (p.workspace) {
    if (p.workspace_bytes < need || reinterpret_cast<uintptr_t>(p.workspace) % kAlign != 0)
      return INFINI_ERR_WORKSPACE;
  }
  rc = check_device(pl.tc);
  if (rc != INFINI_OK) return rc;
  if (pl.tc && !get_encode()) return INFINI_ERR_DEVICE;
  const float scale = p.scale != 0.f ? p.scale : 1.f / sqrtf((float)p.dk);
  char* ws = static_cast<char*>(p.workspace);
  bool own = false;
  if (!ws) {
    void* w = nullptr;
    if (!ws_alloc(&w, need, p.stream)) return INFINI_ERR_WORKSPACE;
    ws = static_cast<char*>(w);
    own = true;
  }
  LocalQK loc;
  memset(&loc, 0, sizeof(loc));
  loc.q = p.q;
  loc.k = p.k;
  for (int i = 0; i < 3; ++i) {
    loc.qs[i] = p.q_stride[i];
    loc.ks[i] = p.k_stride[i];
  }
  rc = rope ? run_rope(p, ws + pl.total, &loc) : INFINI_OK;
  if (rc != INFINI_OK) {
  } else if (pl.tc)
    rc = run_tc(p, pl, ws, scale, loc);
  else if (pl.f32)
    rc = run_simt<float>(p, pl, ws, scale, loc);
  else
    rc = run_simt<__nv_bfloat16>(p, pl, ws, scale, loc);
  if (own && cudaFreeAsync(ws, p.stream) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_WORKSPACE;
  return rc;
}

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  // Nothing arrives on this barrier: the wait must give up after limit_ns.
  mbar_wait(b, 0, limit_ns);
}

// ------------------------------------------------------------ backward
// Workspace of the backward: the forward's CUDA-core plan (fp32 snapshots of
// M^(s), z^(s)), a copy of the running state, the forward's output, A_dot and
// lse, the per-row terms, the partials of the memory-gradient chain, its
// snapshots (linear) or running value (delta), and the update's dk, dv terms.
struct BwdPlan {
  Plan fwd;
  bool tc;  // tensor-core local-attention gradients (bf16, dk = dv = 128)
  int Gc, cpbc, Gu, cpbu;
  size_t off_fwd, off_state, off_out, off_adot, off_lse, off_D, off_brow, off_dden, off_ddenr, off_dnum, off_dnumr,
      off_cpart, off_upart, off_g, off_dkupd, off_dvupd, off_snap32, off_dqmem, total;
};

int bwd_plan(const infini_attn_bwd_params& p, BwdPlan* bp) {
  if (p.B <= 0 || p.H <= 0 || p.L <= 0 || p.N <= 0 || p.d_k <= 0 || p.d_v <= 0) return INFINI_ERR_INVALID_ARG;
  int rc = make_plan(p.B, p.H, p.L, p.N, p.d_k, p.d_v, p.mode, p.flags & INFINI_FLAG_FORCE_SIMT, &bp->fwd);
  if (rc != INFINI_OK) return rc;
  bp->tc = bp->fwd.tc;
  if (!bp->tc && !(p.flags & INFINI_FLAG_FORCE_SIMT)) {
    rc = make_plan(p.B, p.H, p.L, p.N, p.d_k, p.d_v, p.mode, INFINI_FLAG_FORCE_SIMT, &bp->fwd);
    if (rc != INFINI_OK) return rc;
  }
  const Plan& f = bp->fwd;
  const long long BH = (long long)p.B * p.H, rows = BH * p.L;
  if (rows >= (1LL << 40)) return INFINI_ERR_UNSUPPORTED;
  const size_t E = (size_t)p.d_k * p.d_v, es = f.f32 ? 4 : 2;
  const int chunks = (int)((std::min<long long>(p.N, p.L) + kChunk - 1) / kChunk);
  auto groups = [&](long long units, int* cpb) {
    long long c = (units * chunks + kTargetCtas - 1) / kTargetCtas;
    c = std::max<long long>(1, std::min<long long>(c, chunks));
    *cpb = (int)c;
    return (int)((chunks + c - 1) / c);
  };
  bp->Gc = groups(BH * f.S, &bp->cpbc);
  bp->Gu = groups(BH, &bp->cpbu);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  bp->off_fwd = take(f.total);
  bp->off_state = take((size_t)BH * (E + p.d_k) * 4);
  bp->off_out = take((size_t)rows * p.d_v * es);
  bp->off_adot = take((size_t)rows * p.d_v * 4);
  bp->off_lse = take((size_t)rows * 4);
  bp->off_D = take((size_t)rows * 4);
  bp->off_brow = take((size_t)rows * 4);
  bp->off_dden = take((size_t)rows * 4);
  bp->off_ddenr = take(f.delta ? (size_t)rows * 4 : 0);
  bp->off_dnum = take((size_t)rows * p.d_v * 4);
  bp->off_dnumr = take(f.delta ? (size_t)rows * p.d_v * 4 : 0);
  bp->off_cpart = take((size_t)BH * f.S * bp->Gc * (E + p.d_k) * 4);
  bp->off_upart = take(f.delta ? (size_t)BH * bp->Gu * (E + p.d_k) * 4 : 0);
  bp->off_g = take((size_t)BH * (f.delta ? 1 : f.S) * (E + p.d_k) * 4);
  bp->off_dkupd = take((size_t)rows * p.d_k * 4);
  bp->off_dvupd = take((size_t)rows * p.d_v * 4);
  bp->off_snap32 = take(bp->tc ? (size_t)BH * f.S * E * 4 : 0);
  bp->off_dqmem = take(bp->tc ? (size_t)rows * p.d_k * 4 : 0);
  bp->total = off;
  return INFINI_OK;
}

template <typename T>
int run_backward(const infini_attn_bwd_params& p, const BwdPlan& bp, char* ws) {
  const Plan& f = bp.fwd;
  const int dk = p.d_k, dv = p.d_v, BH = p.B * p.H;
  const size_t E = (size_t)dk * dv;
  const float scale = p.scale != 0.f ? p.scale : 1.f / sqrtf((float)dk);
  cudaStream_t st = p.stream;
  float* Mst = reinterpret_cast<float*>(ws + bp.off_state);
  float* zst = Mst + (size_t)BH * E;
  // 1. forward again from (M_0, z_0): snapshots of M^(s), z^(s), A_dot, lse
  if ((p.M0 ? cudaMemcpyAsync(Mst, p.M0, (size_t)BH * E * 4, cudaMemcpyDeviceToDevice, st)
            : cudaMemsetAsync(Mst, 0, (size_t)BH * E * 4, st)) != cudaSuccess ||
      (p.z0 ? cudaMemcpyAsync(zst, p.z0, (size_t)BH * dk * 4, cudaMemcpyDeviceToDevice, st)
            : cudaMemsetAsync(zst, 0, (size_t)BH * dk * 4, st)) != cudaSuccess)
    return INFINI_ERR_LAUNCH;
  infini_attn_params fp;
  memset(&fp, 0, sizeof(fp));
  fp.q = p.q; fp.k = p.k; fp.v = p.v; fp.beta = p.beta; fp.M = Mst; fp.z = zst; fp.out = ws + bp.off_out;
  fp.B = p.B; fp.H = p.H; fp.L = p.L; fp.N = p.N; fp.dk = dk; fp.dv = dv; fp.mode = p.mode; fp.stream = st;
  const long long cst[2][3] = {{(long long)p.H * p.L * dk, p.L * dk, dk}, {(long long)p.H * p.L * dv, p.L * dv, dv}};
  for (int i = 0; i < 3; ++i) {
    fp.q_stride[i] = fp.k_stride[i] = cst[0][i];
    fp.v_stride[i] = fp.o_stride[i] = cst[1][i];
  }
  LocalQK loc;
  memset(&loc, 0, sizeof(loc));
  loc.q = p.q; loc.k = p.k;
  for (int i = 0; i < 3; ++i) loc.qs[i] = loc.ks[i] = cst[0][i];
  float* adot = reinterpret_cast<float*>(ws + bp.off_adot);
  float* lse = reinterpret_cast<float*>(ws + bp.off_lse);
  char* fws = ws + bp.off_fwd;
  int rc;
  const float* snapM;
  if (bp.tc) {
    // tensor-core forward: A_dot in bf16, lse in log2 units, fp32 snapshots of M^(s)
    FwdExtra ex;
    ex.snapM32 = reinterpret_cast<float*>(ws + bp.off_snap32);
    ex.adot = adot;
    ex.lse2 = lse;
    rc = run_tc(fp, f, fws, scale, loc, &ex);
    snapM = ex.snapM32;
  } else {
    rc = run_simt<T>(fp, f, fws, scale, loc, adot, lse);
    snapM = reinterpret_cast<const float*>(fws + f.off_snapM);
  }
  if (rc != INFINI_OK) return rc;
  const float* snapz = reinterpret_cast<const float*>(fws + f.off_snapz);
  BwdGeo g;
  g.B = p.B; g.H = p.H; g.S = f.S; g.N = p.N; g.dk = dk; g.dv = dv; g.L = p.L;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* dout = static_cast<const T*>(p.d_out);
  float* Drow = reinterpret_cast<float*>(ws + bp.off_D);
  float* brow = reinterpret_cast<float*>(ws + bp.off_brow);
  float* dden = reinterpret_cast<float*>(ws + bp.off_dden);
  float* dnum = reinterpret_cast<float*>(ws + bp.off_dnum);
  float* ddenr = reinterpret_cast<float*>(ws + bp.off_ddenr);
  float* dnumr = reinterpret_cast<float*>(ws + bp.off_dnumr);
  float* cpart = reinterpret_cast<float*>(ws + bp.off_cpart);
  float* upart = reinterpret_cast<float*>(ws + bp.off_upart);
  float* gst = reinterpret_cast<float*>(ws + bp.off_g);
  float* dkupd = reinterpret_cast<float*>(ws + bp.off_dkupd);
  float* dvupd = reinterpret_cast<float*>(ws + bp.off_dvupd);
  // 2. dq, D, the dbeta row terms, d_num and d_den rows
  const int QT = (p.N + 31) / 32;
  const int bps = (int)((std::min<long long>(p.N, p.L) + 127) / 128);
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  tc::BwdTcArgs ta;
  float* dqmem = reinterpret_cast<float*>(ws + bp.off_dqmem);
  if (bp.tc) {
    if (!encode_bhld(&tm_q, p.q, p.B, p.H, p.L, cst[0]) || !encode_bhld(&tm_k, p.k, p.B, p.H, p.L, cst[0]) ||
        !encode_bhld(&tm_v, p.v, p.B, p.H, p.L, cst[1]) || !encode_bhld(&tm_do, p.d_out, p.B, p.H, p.L, cst[1]))
      return INFINI_ERR_LAUNCH;
    if (set_tc_smem_limits() != INFINI_OK) return INFINI_ERR_LAUNCH;
    // the memory read's backward and D' = dO . A_dot (products on the tensor cores)
    {
      LaunchScope ls(kPhaseBwdMemTc, st);
      tc::bwd_qmem_tc_kernel<<<(unsigned)((long long)BH * f.S * bps), tc::kQmThreads, tc::kQmSmem, st>>>(
          reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(dout), adot, p.beta,
          snapM, snapz, p.B, p.H, f.S, p.N, p.L, bps, dqmem, Drow, brow, dnum, dden);
    }
    memset(&ta, 0, sizeof(ta));
    ta.lse2 = lse; ta.Dp = Drow; ta.beta = p.beta; ta.mem_q = dqmem;
    ta.mem_k = reinterpret_cast<float*>(ws + bp.off_dkupd);
    ta.mem_v = reinterpret_cast<float*>(ws + bp.off_dvupd);
    ta.B = p.B; ta.H = p.H; ta.S = f.S; ta.T = (p.N + 127) / 128; ta.L = p.L; ta.N = p.N;
    ta.scale = scale; ta.scale_log2 = scale * 1.4426950408889634f;
    ta.out0 = static_cast<__nv_bfloat16*>(p.dq);
    LaunchScope ls(kPhaseBwdTc, st);
    tc::bwd_dq_tc_kernel<<<(unsigned)((long long)ta.T * BH * f.S), tc::kBwdThreads, tc::kDQSmem, st>>>(tm_q, tm_k, tm_v,
                                                                                                    tm_do, ta);
  } else {
    const size_t q_smem = (size_t)(32 * (dk + 1) + 32 * dv + 32 * dk + 2 * 32 * dv) * 4;
    cudaFuncSetAttribute(bwd_q_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)q_smem);
    LaunchScope ls(kPhaseBwd, st);
    bwd_q_kernel<T><<<(unsigned)((long long)QT * BH * f.S), 256, q_smem, st>>>(
        q, k, v, dout, p.beta, adot, lse, snapM, snapz, g, scale, QT, static_cast<T*>(p.dq), Drow, brow, dnum, dden);
  }
  // 3. the memory read's partials sigma(Q)^T [d_num | d_den] of every segment
  const size_t outer_smem = (size_t)(64 * kMP + 64 * 130) * 4;
  cudaFuncSetAttribute(bwd_outer_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)outer_smem);
  if (bp.tc) {
    LaunchScope ls(kPhaseBwdMemTc, st);
    tc::bwd_outer_tc_kernel<<<(unsigned)((long long)BH * f.S * bp.Gc), tc::kOtThreads, tc::kOtSmem, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(q), dnum, dden, p.N, p.L, 0, f.S, bp.Gc, bp.cpbc, cpart);
  } else {
    LaunchScope ls(kPhaseBwd, st);
    bwd_outer_kernel<T><<<(unsigned)((long long)BH * f.S * bp.Gc), 256, outer_smem, st>>>(q, dnum, dden, g, dv, 0, f.S,
                                                                                          bp.Gc, bp.cpbc, cpart);
  }
  const dim3 sgrid((unsigned)((E + dk + 255) / 256), BH);
  const size_t pst = E + dk;
  const size_t upd_smem = (size_t)((f.delta ? 2 : 1) * (128 + 64) * kMP + 2 * 128 + 2 * 64) * 4;
  const int bps64 = (int)((std::min<long long>(p.N, p.L) + 63) / 64);  // update terms: 64 rows per block
  cudaFuncSetAttribute(bwd_upd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)upd_smem);
  // 4. the memory-gradient chain and the update's dk, dv terms
  if (!f.delta) {
    {
      LaunchScope ls(kPhaseBwd, st);
      bwd_state_kernel<<<sgrid, 256, 0, st>>>(nullptr, p.dM_S, p.dz_S, cpart, nullptr, dk, dv, f.S, 0, 0, bp.Gc, 0, gst,
                                              p.dM0, p.dz0);
    }
    if (bp.tc) {
      LaunchScope ls(kPhaseBwdMemTc, st);
      tc::bwd_upd_tc_kernel<<<(unsigned)((long long)BH * f.S * bps), tc::kUpThreads, tc::kUpSmem, st>>>(
          reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v), p.B, p.H, f.S, p.N,
          p.L, 0, gst, (long long)pst, (long long)f.S * pst, nullptr, nullptr, dkupd, dvupd, nullptr, nullptr, bps);
    } else {
      LaunchScope ls(kPhaseBwd, st);
      bwd_upd_kernel<T><<<(unsigned)((long long)BH * f.S * bps64), 256, upd_smem, st>>>(
          k, v, g, 0, gst, (long long)pst, (long long)f.S * pst, nullptr, nullptr, dkupd, dvupd, nullptr, nullptr,
          bps64);
    }
  } else {
    {
      LaunchScope ls(kPhaseBwd, st);
      bwd_state_kernel<<<sgrid, 256, 0, st>>>(gst, p.dM_S, p.dz_S, nullptr, nullptr, dk, dv, f.S, 2, 0, bp.Gc, 0,
                                              nullptr, nullptr, nullptr);
    }
    // the reverse steps' launches as programmatic dependents of the one
    // before (each waits for it before touching memory): their launch
    // latency overlaps the previous kernel's tail
    auto dependent = [&](auto kernel, dim3 grid, unsigned block, size_t smem, auto... args) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.gridDim = grid;
      cfg.blockDim = dim3(block);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
      if (e != cudaSuccess) {
        cudaGetLastError();
        note_cuda_error(e);
      }
      return e == cudaSuccess;
    };
    for (int s = f.S - 1; s >= 0; --s) {
      if (bp.tc) {
        LaunchScope ls(kPhaseBwdMemTc, st);
        if (!dependent(tc::bwd_upd_tc_kernel, dim3((unsigned)((long long)BH * bps)), (unsigned)tc::kUpThreads,
                       (size_t)tc::kUpSmem, reinterpret_cast<const __nv_bfloat16*>(k),
                       reinterpret_cast<const __nv_bfloat16*>(v), p.B, p.H, f.S, p.N, p.L, s,
                       static_cast<const float*>(gst), 0LL, (long long)pst, snapM, snapz, dkupd, dvupd, dnumr, ddenr,
                       bps))
          return INFINI_ERR_LAUNCH;
      } else {
        LaunchScope ls(kPhaseBwd, st);
        bwd_upd_kernel<T><<<(unsigned)((long long)BH * bps64), 256, upd_smem, st>>>(
            k, v, g, s, gst, 0, (long long)pst, snapM, snapz, dkupd, dvupd, dnumr, ddenr, bps64);
      }
      if (bp.tc) {
        LaunchScope ls(kPhaseBwdMemTc, st);
        if (!dependent(tc::bwd_outer_tc_kernel, dim3((unsigned)((long long)BH * bp.Gu)), (unsigned)tc::kOtThreads,
                       (size_t)tc::kOtSmem, reinterpret_cast<const __nv_bfloat16*>(k),
                       static_cast<const float*>(dnumr), static_cast<const float*>(ddenr), p.N, p.L, s, 1, bp.Gu,
                       bp.cpbu, upart))
          return INFINI_ERR_LAUNCH;
      } else {
        LaunchScope ls(kPhaseBwd, st);
        bwd_outer_kernel<T><<<(unsigned)((long long)BH * bp.Gu), 256, outer_smem, st>>>(k, dnumr, ddenr, g, dv, s, 1,
                                                                                       bp.Gu, bp.cpbu, upart);
      }
      LaunchScope ls(kPhaseBwd, st);
      if (bp.tc) {
        if (!dependent(bwd_state_kernel, sgrid, 256u, (size_t)0, gst, static_cast<const float*>(nullptr),
                       static_cast<const float*>(nullptr), static_cast<const float*>(cpart),
                       static_cast<const float*>(upart), dk, dv, f.S, 1, s, bp.Gc, bp.Gu, static_cast<float*>(nullptr),
                       static_cast<float*>(nullptr), static_cast<float*>(nullptr)))
          return INFINI_ERR_LAUNCH;
      } else {
        bwd_state_kernel<<<sgrid, 256, 0, st>>>(gst, nullptr, nullptr, cpart, upart, dk, dv, f.S, 1, s, bp.Gc, bp.Gu,
                                                nullptr, nullptr, nullptr);
      }
    }
    LaunchScope ls(kPhaseBwd, st);
    bwd_state_kernel<<<sgrid, 256, 0, st>>>(gst, nullptr, nullptr, nullptr, nullptr, dk, dv, f.S, 3, 0, 0, 0, nullptr,
                                            p.dM0, p.dz0);
  }
  // 5. dk, dv of the local attention plus the update's terms
  if (bp.tc) {
    ta.out0 = static_cast<__nv_bfloat16*>(p.dk);
    ta.out1 = static_cast<__nv_bfloat16*>(p.dv);
    LaunchScope ls(kPhaseBwdTc, st);
    tc::bwd_dkdv_tc_kernel<<<(unsigned)((long long)ta.T * BH * f.S), tc::kBwdThreads, tc::kKVSmem, st>>>(
        tm_q, tm_k, tm_v, tm_do, ta);
  } else {
    const size_t kv_smem = (size_t)(32 * dk + 32 * dv + 32 * (dk + 1) + 32 * (dv + 1) + 64) * 4;
    cudaFuncSetAttribute(bwd_kv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kv_smem);
    LaunchScope ls(kPhaseBwd, st);
    bwd_kv_kernel<T><<<(unsigned)((long long)QT * BH * f.S), 256, kv_smem, st>>>(
        q, k, v, dout, p.beta, lse, Drow, dkupd, dvupd, g, scale, QT, static_cast<T*>(p.dk), static_cast<T*>(p.dv));
  }
  // 6. dbeta
  LaunchScope ls(kPhaseBwd, st);
  bwd_beta_kernel<<<p.H, 256, 0, st>>>(brow, p.beta, p.B, p.H, p.L, p.dbeta);
  return launch_status();
}

int backward_impl(const infini_attn_bwd_params& p) {
  if (!p.q || !p.k || !p.v || !p.beta || !p.d_out || !p.dq || !p.dk || !p.dv || !p.dbeta) return INFINI_ERR_INVALID_ARG;
  BwdPlan bp;
  int rc = bwd_plan(p, &bp);
  if (rc != INFINI_OK) return rc;
  const bool f32 = bp.fwd.f32;
  const size_t es = f32 ? 4 : 2;
  const long long BH = (long long)p.B * p.H;
  const size_t nq = (size_t)BH * p.L * p.d_k * es, nv = (size_t)BH * p.L * p.d_v * es;
  // outputs must not overlap the inputs or one another
  const void* outs[3] = {p.dq, p.dk, p.dv};
  const size_t outn[3] = {nq, nq, nv};
  const void* ins[4] = {p.q, p.k, p.v, p.d_out};
  const size_t inn[4] = {nq, nq, nv, nv};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 4; ++b)
      if (ranges_overlap(outs[a], outn[a], ins[b], inn[b])) return INFINI_ERR_INVALID_ARG;
    for (int b = a + 1; b < 3; ++b)
      if (ranges_overlap(outs[a], outn[a], outs[b], outn[b])) return INFINI_ERR_INVALID_ARG;
  }
  if (bp.tc) {
    const void* ptrs[7] = {p.q, p.k, p.v, p.d_out, p.dq, p.dk, p.dv};
    bool aligned = true;
    for (const void* x : ptrs) aligned = aligned && reinterpret_cast<uintptr_t>(x) % 16 == 0;
    if (!aligned) {  // TMA needs 16-byte aligned rows: the CUDA-core kernels take the call
      infini_attn_bwd_params q2 = p;
      q2.flags |= INFINI_FLAG_FORCE_SIMT;
      return backward_impl(q2);
    }
  }
  if (p.workspace && (p.workspace_bytes < bp.total || reinterpret_cast<uintptr_t>(p.workspace) % kAlign != 0))
    return INFINI_ERR_WORKSPACE;
  rc = check_device(false);
  if (rc != INFINI_OK) return rc;
  char* ws = static_cast<char*>(p.workspace);
  bool own = false;
  if (!ws) {
    void* w = nullptr;
    if (!ws_alloc(&w, bp.total, p.stream)) return INFINI_ERR_WORKSPACE;
    ws = static_cast<char*>(w);
    own = true;
  }
  rc = f32 ? run_backward<float>(p, bp, ws) : run_backward<__nv_bfloat16>(p, bp, ws);
  if (own && cudaFreeAsync(ws, p.stream) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_WORKSPACE;
  return rc;
}

// ------------------------------------------------------------ fixed scratch
// Workspace of infini_attn_forward_noalloc: one buffer per device, part of
// the module image, so it exists from load to exit and no call allocates.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the buffer in the current context.  The symbol's name is
// only a host-side handle; the address comes from cudaGetSymbolAddress, once
// per context (so once per device while its context lives), with that
// device current.  Keyed by context id: after a device reset the address is
// looked up again instead of reusing one from the destroyed context.
int noalloc_scratch(void** out) {
  static std::mutex mu;
  static std::vector<std::pair<unsigned long long, void*>> addr;
  std::lock_guard<std::mutex> lk(mu);
  unsigned long long ctx = current_context_id();
  for (const auto& e : addr)
    if (ctx != 0 && e.first == ctx) {
      *out = e.second;
      return INFINI_OK;
    }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return INFINI_ERR_LAUNCH;
  }
  // the lookup made the device's primary context current if none was
  ctx = current_context_id();
  if (ctx != 0) addr.emplace_back(ctx, p);
  *out = p;
  return INFINI_OK;
}

}  // namespace
}  // namespace infini

using namespace infini;

// ------------------------------------------------------------------ full layer
// Q, K, V = X W_{Q,K,V}, the Infini-attention forward, Y = A W_O (multi-head
// formulation, Eq. 5 and Eq. 11).  The projections run on the library's own
// tcgen05 GEMM (gemm_tc_kernel); the layout keeps them copy-free: the QKV product [B*L, 3*H*128] is read by
// the attention kernels through strided views, and the attention writes its
// output as [B, L, H, 128], the A operand of the output projection.
namespace {

constexpr int kLayerHead = 128;

struct LayerPlan {
  size_t off_qkv, off_ao, off_attn, attn_bytes, total;
  long long rows;  // B * L
};

bool layer_plan(int B, int H, long long L, int N, int d_model, int mode, LayerPlan* lp) {
  if (B <= 0 || H <= 0 || L <= 0 || N <= 0 || d_model <= 0) return false;
  if ((mode & ~INFINI_DELTA) != 0) return false;  // bf16 layer: no INFINI_F32
  const long long rows = (long long)B * L;
  if (rows > (1LL << 31) - 1 || 3LL * H * kLayerHead > (1LL << 31) - 1) return false;
  const size_t attn = infini_attn_workspace_size(B, H, (long)L, N, kLayerHead, kLayerHead, mode);
  if (attn == 0) return false;
  size_t off = 0;
  lp->off_qkv = off;
  off = align_up(off + (size_t)rows * 3 * H * kLayerHead * 2);
  lp->off_ao = off;
  off = align_up(off + (size_t)rows * H * kLayerHead * 2);
  lp->off_attn = off;
  lp->attn_bytes = attn;
  lp->total = align_up(off + attn);
  lp->rows = rows;
  return true;
}

int decode_fold(void* k_cache, void* v_cache, const float* beta, float* M, float* z, int B, int H, int N, int n,
                int dk, int dv, int mode, cudaStream_t stream);

}  // namespace

extern "C" {

int infini_attn_forward(const void* q, const void* k, const void* v, const float* beta, float* M, float* z, void* out,
                        int B, int H, long L, int N, int dk, int dv, int mode, cudaStream_t stream) {
  infini_attn_params p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.M = M; p.z = z; p.out = out;
  p.B = B; p.H = H; p.L = L; p.N = N; p.dk = dk; p.dv = dv; p.mode = mode; p.stream = stream;
  return forward_impl(p);
}

int infini_attn_segment_step(const void* q, const void* k, const void* v, const float* beta, float* M, float* z,
                             void* out, int B, int H, int n, int dk, int dv, int mode, cudaStream_t stream) {
  if (n <= 0) return INFINI_ERR_INVALID_ARG;
  return infini_attn_forward(q, k, v, beta, M, z, out, B, H, n, n, dk, dv, mode, stream);
}

int infini_attn_forward_noalloc(const void* q, const void* k, const void* v, const float* beta, float* M, float* z,
                                void* out, int B, int H, long L, int N, int dk, int dv, int mode,
                                cudaStream_t stream) {
  if (!q || !k || !v || !beta || !M || !z || !out) return INFINI_ERR_INVALID_ARG;
  Plan pl;
  int rc = make_plan(B, H, L, N, dk, dv, mode, 0, &pl);
  if (rc != INFINI_OK) return rc;
  // the documented limit: infini_attn_workspace_size, which also covers the
  // CUDA-core kernels a misaligned layout falls back to
  if (infini_attn_workspace_size(B, H, L, N, dk, dv, mode) > kNoAllocScratchBytes) return INFINI_ERR_SCRATCH_LIMIT;
  rc = check_device(pl.tc);
  if (rc != INFINI_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != INFINI_OK) return rc;
  infini_attn_params p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.beta = beta; p.M = M; p.z = z; p.out = out;
  p.B = B; p.H = H; p.L = L; p.N = N; p.dk = dk; p.dv = dv; p.mode = mode; p.stream = stream;
  p.workspace = scratch;
  p.workspace_bytes = kNoAllocScratchBytes;
  return forward_impl(p);
}

int infini_attn_forward_ex(const infini_attn_params* p) {
  if (!p) return INFINI_ERR_INVALID_ARG;
  return forward_impl(*p);
}

size_t infini_attn_workspace_size(int B, int H, long L, int N, int dk, int dv, int mode) {
  Plan pl;
  if (make_plan(B, H, L, N, dk, dv, mode, 0, &pl) != INFINI_OK) return 0;
  Plan pl2;  // a layout that falls back to CUDA cores needs the fp32 snapshots
  if (make_plan(B, H, L, N, dk, dv, mode, INFINI_FLAG_FORCE_SIMT, &pl2) != INFINI_OK) return 0;
  return std::max(pl.total, pl2.total);
}


int infini_attn_backward(const infini_attn_bwd_params* p) {
  if (!p) return INFINI_ERR_INVALID_ARG;
  return backward_impl(*p);
}

size_t infini_attn_backward_workspace_size(const infini_attn_bwd_params* p) {
  if (!p) return 0;
  BwdPlan bp, bs;
  if (bwd_plan(*p, &bp) != INFINI_OK) return 0;
  // a call whose tensors are not 16-byte aligned runs on the CUDA cores, whose plan may be larger
  infini_attn_bwd_params q = *p;
  q.flags |= INFINI_FLAG_FORCE_SIMT;
  if (bwd_plan(q, &bs) != INFINI_OK) return 0;
  return std::max(bp.total, bs.total);
}

size_t infini_attn_workspace_size_ex(const infini_attn_params* p) {
  if (!p) return 0;
  if (p->rope_base != 0.0 && !(p->rope_base > 0.0 && std::isfinite(p->rope_base) && p->dk % 2 == 0)) return 0;
  const size_t base = infini_attn_workspace_size(p->B, p->H, (long)p->L, p->N, p->dk, p->dv, p->mode);
  return base == 0 ? 0 : base + rope_bytes(*p);
}

int infini_attn_decode_step(const void* q_t, const void* k_t, const void* v_t, void* k_cache, void* v_cache,
                            const float* beta, float* M, float* z, void* out, int B, int H, int N, int pos, int dk,
                            int dv, int mode, int fold, cudaStream_t stream) {
  if (!q_t || !k_t || !v_t || !k_cache || !v_cache || !beta || !M || !z || !out) return INFINI_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || dk <= 0 || dv <= 0 || pos < 0 || pos >= N) return INFINI_ERR_INVALID_ARG;
  if ((mode & ~(INFINI_DELTA | INFINI_F32)) != 0 || dk > 128 || dv > 128) return INFINI_ERR_UNSUPPORTED;
  const bool f32 = (mode & INFINI_F32) != 0;
  const long long BH = (long long)B * H;
  if (BH > (1LL << 31) - 1) return INFINI_ERR_UNSUPPORTED;
  int rc = check_device(false);
  if (rc != INFINI_OK) return rc;
  const int n = pos + 1;
  const float scale = 1.f / sqrtf((float)dk);
  // 1 + 2. the token's output, its key and value appended to the caches by the
  // same launch: one thread-block cluster per (b, h) over up to 8 key ranges
  // of at least 64 keys, merged through distributed shared memory
  if (BH <= 65535) {
    const long long want =
        std::max<long long>(1, std::min<long long>(kDecodeMaxSplits, (2LL * kSms + BH - 1) / BH));
    int per = (int)std::max<long long>(64, (n + want - 1) / want);
    int splits = (n + per - 1) / per;  // <= 16: a non-portable cluster size beyond 8
    // 16-byte row loads: rows of a multiple of 16 bytes, 16-byte aligned bases
    const size_t es = f32 ? 4 : 2;
    const int vec = ((size_t)dk * es) % 16 == 0 && reinterpret_cast<uintptr_t>(k_cache) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(k_t) % 16 == 0;
    {
      static std::mutex mu;
      static std::vector<unsigned long long> done;  // contexts with the cluster-size attribute set
      const unsigned long long ctx = current_context_id();
      std::lock_guard<std::mutex> lk(mu);
      if (ctx == 0 || std::find(done.begin(), done.end(), ctx) == done.end()) {
        if (cudaFuncSetAttribute(decode_fused_kernel<float>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode_fused_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
          cudaGetLastError();
          return INFINI_ERR_LAUNCH;
        }
        if (ctx != 0) done.push_back(ctx);
      }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)splits, (unsigned)BH);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaSuccess;
    for (int attempt = 0; attempt < 2; ++attempt) {
      if (attempt == 1) {
        // a 16-CTA cluster could not be placed: ranges for clusters of at most 8
        if (splits <= 8) break;
        cudaGetLastError();
        per = std::max(64, (n + 7) / 8);
        splits = (n + per - 1) / per;
        attr[0].val.clusterDim.x = (unsigned)splits;
        cfg.gridDim = dim3((unsigned)splits, (unsigned)BH);
      }
      LaunchScope ls(kPhaseAttn, stream);
      if (f32)
        e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<float>, static_cast<const float*>(q_t),
                               static_cast<const float*>(k_t), static_cast<const float*>(v_t),
                               static_cast<float*>(k_cache), static_cast<float*>(v_cache), beta, (const float*)M,
                               (const float*)z, static_cast<float*>(out), H, N, n, dk, dv, scale, per, vec);
      else
        e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(q_t),
                               static_cast<const __nv_bfloat16*>(k_t), static_cast<const __nv_bfloat16*>(v_t),
                               static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), beta,
                               (const float*)M, (const float*)z, static_cast<__nv_bfloat16*>(out), H, N, n, dk, dv,
                               scale, per, vec);
      if (e == cudaSuccess) break;
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      return note_cuda_error(e);
    }
    if (!(fold || pos == N - 1)) return INFINI_OK;
    return decode_fold(k_cache, v_cache, beta, M, z, B, H, N, n, dk, dv, mode, stream);
  }
  // more (b, h) than a grid's second dimension holds: ranges on the second
  // dimension, partial states in a scratch buffer, a second launch merges
  const long long want = std::max<long long>(1, (2LL * kSms + BH - 1) / BH);
  int per = (int)std::max<long long>(64, (n + want - 1) / want);
  const int splits = (n + per - 1) / per;
  void* scratch = nullptr;
  if (!ws_alloc(&scratch, (size_t)splits * BH * (dv + 2) * 4, stream)) return INFINI_ERR_WORKSPACE;
  float* part = static_cast<float*>(scratch);
  {
    LaunchScope ls(kPhaseAttn, stream);
    const dim3 grid((unsigned)BH, (unsigned)splits);
    if (f32)
      decode_part_kernel<float><<<grid, 256, 0, stream>>>(
          static_cast<const float*>(q_t), static_cast<const float*>(k_t), static_cast<const float*>(v_t),
          static_cast<float*>(k_cache), static_cast<float*>(v_cache), N, n, dk, dv, scale, per, part);
    else
      decode_part_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(q_t), static_cast<const __nv_bfloat16*>(k_t),
          static_cast<const __nv_bfloat16*>(v_t), static_cast<__nv_bfloat16*>(k_cache),
          static_cast<__nv_bfloat16*>(v_cache), N, n, dk, dv, scale, per, part);
  }
  {
    LaunchScope ls(kPhaseAttn, stream);
    if (f32)
      decode_merge_kernel<float><<<(unsigned)BH, 128, 0, stream>>>(static_cast<const float*>(q_t), beta, M, z, part,
                                                                    splits, H, dk, dv, static_cast<float*>(out));
    else
      decode_merge_kernel<__nv_bfloat16><<<(unsigned)BH, 128, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(q_t), beta, M, z, part, splits, H, dk, dv,
          static_cast<__nv_bfloat16*>(out));
  }
  rc = launch_status();
  if (cudaFreeAsync(scratch, stream) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_WORKSPACE;
  if (rc != INFINI_OK || !(fold || pos == N - 1)) return rc;
  return decode_fold(k_cache, v_cache, beta, M, z, B, H, N, n, dk, dv, mode, stream);
}

}  // extern "C"

namespace {
// 3. the segment is complete: fold its n keys and values into M, z with the
// forward's update kernels alone (no attention, no output).
int decode_fold(void* k_cache, void* v_cache, const float* beta, float* M, float* z, int B, int H, int N, int n,
                int dk, int dv, int mode, cudaStream_t stream) {
  infini_attn_params p;
  memset(&p, 0, sizeof(p));
  p.q = k_cache;
  p.k = k_cache;
  p.v = v_cache;
  p.beta = beta;
  p.M = M;
  p.z = z;
  p.out = nullptr;
  p.B = B;
  p.H = H;
  p.L = n;
  p.N = n;
  p.dk = dk;
  p.dv = dv;
  p.mode = mode;
  p.flags = kFlagUpdateOnly;
  const long long ks[3] = {(long long)H * N * dk, (long long)N * dk, dk};
  const long long vs[3] = {(long long)H * N * dv, (long long)N * dv, dv};
  for (int i = 0; i < 3; ++i) {
    p.q_stride[i] = p.k_stride[i] = ks[i];
    p.v_stride[i] = vs[i];
    p.o_stride[i] = vs[i];
  }
  p.stream = stream;
  return forward_impl(p);
}
}  // namespace

extern "C" {

int infini_attn_gemm_bf16(const void* A, const void* Bm, void* C, long M, int N, int K, cudaStream_t stream) {
  if (!A || !Bm || !C) return INFINI_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return INFINI_ERR_INVALID_ARG;
  if (ranges_overlap(C, (size_t)M * N * 2, A, (size_t)M * K * 2) || ranges_overlap(C, (size_t)M * N * 2, Bm, (size_t)K * N * 2))
    return INFINI_ERR_INVALID_ARG;
  if (N % 8 || K % 8) return INFINI_ERR_UNSUPPORTED;
  const int rc = check_device(true);
  if (rc != INFINI_OK) return rc;
  return gemm_tc(A, K, Bm, N, C, N, M, N, K, stream);
}

size_t infini_attn_layer_workspace_size(int B, int H, long L, int N, int d_model, int mode) {
  LayerPlan lp;
  return layer_plan(B, H, L, N, d_model, mode, &lp) ? lp.total : 0;
}

int infini_attn_layer_forward(const void* x, const void* w_qkv, const void* w_o, const float* beta, float* M,
                              float* z, void* y, int B, int H, long L, int N, int d_model, int mode, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  if (!x || !w_qkv || !w_o || !beta || !M || !z || !y) return INFINI_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || L <= 0 || N <= 0 || d_model <= 0) return INFINI_ERR_INVALID_ARG;
  LayerPlan lp;
  if (!layer_plan(B, H, L, N, d_model, mode, &lp)) return INFINI_ERR_UNSUPPORTED;
  const size_t ybytes = (size_t)lp.rows * d_model * 2;
  if (ranges_overlap(y, ybytes, x, ybytes) || ranges_overlap(y, ybytes, w_qkv, (size_t)d_model * 3 * H * kLayerHead * 2) ||
      ranges_overlap(y, ybytes, w_o, (size_t)H * kLayerHead * d_model * 2))
    return INFINI_ERR_INVALID_ARG;
  if (workspace && (workspace_bytes < lp.total || reinterpret_cast<uintptr_t>(workspace) % kAlign != 0))
    return INFINI_ERR_WORKSPACE;
  if (d_model % 8 != 0 || reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(w_qkv) % 16 ||
      reinterpret_cast<uintptr_t>(w_o) % 16 || reinterpret_cast<uintptr_t>(y) % 16)
    return INFINI_ERR_UNSUPPORTED;
  int rc = check_device(true);
  if (rc != INFINI_OK) return rc;
  char* ws = static_cast<char*>(workspace);
  bool own = false;
  if (!ws) {
    void* w = nullptr;
    if (!ws_alloc(&w, lp.total, stream)) return INFINI_ERR_WORKSPACE;
    ws = static_cast<char*>(w);
    own = true;
  }
  const long long HD = (long long)H * kLayerHead;
  __nv_bfloat16* qkv = reinterpret_cast<__nv_bfloat16*>(ws + lp.off_qkv);
  __nv_bfloat16* ao = reinterpret_cast<__nv_bfloat16*>(ws + lp.off_ao);
  rc = gemm_tc(x, d_model, w_qkv, 3 * HD, qkv, 3 * HD, lp.rows, 3 * HD, d_model, stream);
  if (rc == INFINI_OK) {
    infini_attn_params p;
    memset(&p, 0, sizeof(p));
    p.q = qkv;
    p.k = qkv + HD;
    p.v = qkv + 2 * HD;
    p.beta = beta;
    p.M = M;
    p.z = z;
    p.out = ao;
    p.B = B;
    p.H = H;
    p.L = L;
    p.N = N;
    p.dk = p.dv = kLayerHead;
    p.mode = mode;
    // views of the [B*L, 3*H*128] product: (B, H, L) strides
    const long long in_st[3] = {(long long)L * 3 * HD, kLayerHead, 3 * HD};
    const long long out_st[3] = {(long long)L * HD, kLayerHead, HD};
    for (int i = 0; i < 3; ++i) {
      p.q_stride[i] = p.k_stride[i] = p.v_stride[i] = in_st[i];
      p.o_stride[i] = out_st[i];
    }
    p.workspace = ws + lp.off_attn;
    p.workspace_bytes = lp.attn_bytes;
    p.stream = stream;
    rc = forward_impl(p);
  }
  if (rc == INFINI_OK) rc = gemm_tc(ao, HD, w_o, d_model, y, d_model, lp.rows, d_model, HD, stream);
  if (own && cudaFreeAsync(ws, stream) != cudaSuccess && rc == INFINI_OK) rc = INFINI_ERR_WORKSPACE;
  return rc;
}

int infini_attn_trim_workspace(void) {
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_pool_mu);
  for (const auto& e : g_pools)
    if (e.first == ctx && cudaMemPoolTrimTo(e.second, 0) != cudaSuccess) {
      cudaGetLastError();
      return INFINI_ERR_DEVICE;
    }
  return INFINI_OK;
}
const char* infini_attn_error_string(int code) {
  switch (code) {
    case INFINI_OK: return "ok";
    case INFINI_ERR_INVALID_ARG: return "invalid argument (null pointer, non-positive size, or aliasing buffers)";
    case INFINI_ERR_UNSUPPORTED: return "unsupported head size, mode, layout or size";
    case INFINI_ERR_WORKSPACE: return "workspace too small, misaligned, or allocation failed";
    case INFINI_ERR_LAUNCH: return "CUDA launch or runtime call failed";
    case INFINI_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case INFINI_ERR_DEVICE: return "no usable CUDA device (sm_100 required)";
    case INFINI_ERR_SCRATCH_LIMIT:
      return "shape needs more workspace than the 32 MiB fixed scratch of infini_attn_forward_noalloc";
    default: return "unknown error code";
  }
}

int infini_attn_device_status(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return INFINI_ERR_LAUNCH;
  unsigned st = 0;
  if (cudaMemcpyFromSymbol(&st, g_status, sizeof(st)) != cudaSuccess) return INFINI_ERR_LAUNCH;
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return INFINI_ERR_LAUNCH;
  }
  return (st & kStatusTimeout) ? INFINI_ERR_TIMEOUT : INFINI_OK;
}

int infini_attn_selftest_timeout(unsigned limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return INFINI_ERR_INVALID_ARG;
  int rc = check_device(false);
  if (rc != INFINI_OK) return rc;
  selftest_wait_kernel<<<1, 1, 0, stream>>>((unsigned long long)limit_us * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return INFINI_ERR_LAUNCH;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return INFINI_ERR_LAUNCH;
  return infini_attn_device_status(0);
}

int infini_attn_path(int dk, int dv, int mode, int flags) {
  Plan pl;
  int rc = make_plan(1, 1, 1, 1, dk, dv, mode, flags, &pl);
  if (rc != INFINI_OK) return rc;
  return pl.tc ? 1 : 0;
}

size_t infini_attn_params_size(void) { return sizeof(infini_attn_params); }

#ifdef INFINI_ATTN_TRACE
// Tuning builds only: copies the attention pipeline timestamps to the host.
INFINI_API int infini_attn_debug_trace(unsigned long long* host, int n) {
  if (cudaDeviceSynchronize() != cudaSuccess) return INFINI_ERR_LAUNCH;
  return cudaMemcpyFromSymbol(host, tc::g_attn_trace, sizeof(unsigned long long) * std::min(n, 4096)) == cudaSuccess
             ? INFINI_OK
             : INFINI_ERR_LAUNCH;
}
#endif

int infini_attn_profile_enable(int phase_mask) {
  if (phase_mask < 0 || phase_mask >= (1 << kPhases)) return INFINI_ERR_INVALID_ARG;
  g_profile_mask.store(phase_mask);
  return INFINI_OK;
}

int infini_attn_profile_read(double* ms, long long* launches, int reset) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int rc = INFINI_OK;
  double acc[kPhases] = {};
  long long cnt[kPhases] = {};
  for (const EventPair& e : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(e.b) != cudaSuccess || cudaEventElapsedTime(&t, e.a, e.b) != cudaSuccess) {
      rc = INFINI_ERR_LAUNCH;
      continue;
    }
    acc[e.phase] += t;
    cnt[e.phase] += 1;
  }
  for (int i = 0; i < kPhases; ++i) {
    if (ms) ms[i] += acc[i];
    if (launches) launches[i] += cnt[i];
  }
  if (reset) {
    for (const EventPair& e : g_prof) {
      if (e.ctx != 0) {  // back to the pool of their context
        g_event_pool.emplace_back(e.ctx, e.a);
        g_event_pool.emplace_back(e.ctx, e.b);
      } else {
        cudaEventDestroy(e.a);
        cudaEventDestroy(e.b);
      }
    }
    g_prof.clear();
  }
  return rc;
}

long long infini_attn_launch_count(void) { return g_launches.load(); }

int infini_attn_last_cuda_error(char* name, int n) {
  const int e = g_last_cuda_error.load();
  if (name != nullptr && n > 0) {
    const char* s = e != 0 ? cudaGetErrorName((cudaError_t)e) : "cudaSuccess";
    std::snprintf(name, (size_t)n, "%s", s != nullptr ? s : "unknown");
  }
  return e;
}

}  // extern "C"
