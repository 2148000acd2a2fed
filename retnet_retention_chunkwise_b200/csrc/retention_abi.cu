// retention_abi.cu -- the C ABI of libretention (declared in include/retention.h):
// argument validation, TMA descriptor encoding, launch configuration.
//
// The whole library is this one translation unit (the kernels live in the
// included .cuh files), so the device status word has a single definition.
// No function here allocates memory; every launch goes to the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/retention.h"
#include "chunkwise_tc.cuh"
#include "chunkwise_wide.cuh"
#include "groupnorm.cuh"
#include "backward.cuh"
#include "decode.cuh"
#include "parallel_tc.cuh"
#include "simt_f32.cuh"
#include "state_fold.cuh"
#include "tc_common.cuh"

namespace {

using namespace ret;

// An NVTX range around each compute call of the C ABI, named after the call,
// so a profiler's timeline shows which library call launched which kernels.
// Without a profiler attached the push and pop return at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Wall-clock budget of any single wait inside a kernel.  A healthy wait is
// microseconds; this only bounds a kernel whose pipeline broke.
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s
constexpr uint32_t kWaitIter = 1u << 24;      // polls (each parks for at most 100 us)

// RETENTION_WAIT_LIMIT_MS (read at every launch) shortens or lengthens it.
WaitLimit wait_limit() {
  WaitLimit w{kWaitNs, kWaitIter};
  const char* e = getenv("RETENTION_WAIT_LIMIT_MS");
  const int ms = e ? atoi(e) : 0;
  if (ms > 0) w.ns = (uint64_t)ms * 1000000ull;
  return w;
}

// Fault injection for tests of the bounded-wait path: with
// RETENTION_DEBUG_DROP_BLOCK=n (read at every launch) the chunkwise kernels
// never issue the K load of block n, so the wait for it expires, the kernel
// tears down and the device status reads RET_ETIMEOUT.  Unset: -1, no effect.
int debug_drop_block() {
  const char* e = getenv("RETENTION_DEBUG_DROP_BLOCK");
  return e ? atoi(e) : -1;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 view [n_heads][rows][inner] with a 64 x box_rows box, 128-byte swizzle.
// Rows past the end of a head read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int inner, int rows, int n_heads, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)n_heads};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * rows * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ret_status check_gamma(const float* gamma, int H) {
  if (!gamma) return RET_EINVAL;
  for (int h = 0; h < H; ++h)
    if (!(gamma[h] >= 0.f && gamma[h] <= 1.f)) return RET_EINVAL;  // also rejects NaN
  return RET_OK;
}

ret_status check_shape(const ret_shape& s, bool need_L) {
  if (s.B < 1 || s.H < 1 || s.dk < 1 || s.dv < 1) return RET_EINVAL;
  if (need_L && s.L < 0) return RET_EINVAL;
  if (s.H > RET_MAX_HEADS) return RET_EUNSUPPORTED;
  if ((long long)s.B * s.H > 65535) return RET_EUNSUPPORTED;  // grid.y / grid.z limit
  return RET_OK;
}

// Tensor-core path requires an sm_100 device.
bool device_is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

int max_smem_optin() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return v;
}

float log2_gamma(float g) {
  // log2 in double, rounded once; gamma = 0 -> -inf so gamma^n = exp2(-inf) = 0 for n >= 1
  return g == 0.f ? -INFINITY : (float)std::log2((double)g);
}

void fill_l2g(CwDecay& d, const float* gamma, int H) {
  for (int h = 0; h < H; ++h) d.l2g[h] = log2_gamma(gamma[h]);
}

ret_status launch_status() { return cudaGetLastError() == cudaSuccess ? RET_OK : RET_ECUDA; }

// Launch that may start while the previous launch on the stream is still
// running (programmatic dependent launch).  The kernel must call griddep_wait
// before it touches memory that launch writes or reads.
template <typename... KArgs, typename... Args>
ret_status launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? RET_OK : RET_ECUDA;
}

bool tc_shape_ok(const ret_shape& s) {
  return (s.dk == 64 || s.dk == 128 || s.dk == 256) && (s.dv % kCW_DVT) == 0;
}

// Shapes of the bf16 parallel path: dk in {64, 128, 256}, dv a multiple of 64.
bool parallel_tc_shape_ok(const ret_shape& s) {
  return (s.dk == 64 || s.dk == 128 || s.dk == 256) && s.dv % 64 == 0;
}

// Block lengths of the bf16 chunkwise path: multiples of 16 up to 128 for
// every dk; up to 256 for dk <= 128 (two row halves per block).
bool tc_chunk_ok(int chunk, int dk) {
  return chunk >= 16 && chunk % 16 == 0 && (chunk <= 128 || (chunk <= 256 && dk <= 128));
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Sequence split for the chunkwise tensor-core path: enough segments to give
// every SM a CTA, each segment at least two blocks long.
void plan_segments(const ret_shape& s, int C, int* n_seg, int* seg_chunks) {
  const int n_chunks = (s.L + C - 1) / C;
  const long long base = (long long)(s.dv / kCW_DVT) * s.B * s.H;
  int g = 1;
  if (base < sm_count()) g = (int)(sm_count() / base);
  g = std::max(1, std::min(g, n_chunks / 2));
  const int sc = (n_chunks + g - 1) / g;
  *seg_chunks = std::max(sc, 1);
  *n_seg = (n_chunks + *seg_chunks - 1) / *seg_chunks;
}

size_t seg_workspace_bytes(const ret_shape& s, int n_seg) {
  if (n_seg <= 1) return 0;
  return (size_t)s.B * s.H * n_seg * (size_t)s.dk * s.dv * sizeof(float);
}

// Sequence-split plan of one chunkwise call: n_seg segments of seg_chunks
// blocks (the last may be shorter).
struct SegPlan {
  int n_seg, seg_chunks;
};

// Segment states taken from another anti-causal sum whose state is the
// transpose of this one's (the two anti-causal sums of the backward pass):
// its scanned workspace [BH][n_src][dv][dk], its segments `step` times
// shorter than this call's (plan).
struct SegReuse {
  const float* src;
  int n_src, step;
  SegPlan plan;
};

// Group normalisation in the chunkwise epilogue (see CwArgs::gn).
struct GnParams {
  float eps;
  const float* weight;
  const float* bias;
};

// REV = true runs the anti-causal sum (see chunkwise_dir); blocks longer than
// 128 rows have no anti-causal kernel.  gn: normalise y in the epilogue (the
// causal dk <= 128 kernel with one dv slice per head).  force: use this sequence-split plan
// instead of the default one (still reduced if the workspace is short);
// used: the plan run; reuse: no segment-sum pass of its own (dk <= 128
// anti-causal kernel only).
template <int DK, bool REV>
ret_status launch_chunkwise_tc(const void* q, const void* k, const void* v, const float* gamma,
                               void* y, const float* state_in, float* state_out, int C,
                               const ret_shape& s, void* ws, size_t ws_bytes, cudaStream_t st,
                               const SegPlan* force = nullptr, SegPlan* used = nullptr,
                               const SegReuse* reuse = nullptr, const GnParams* gn = nullptr) {
  if (reuse && (!REV || DK > 128 || C > 128)) return RET_EINVAL;
  if (gn && (REV || DK > 128 || C > 128 || s.dv != kCW_DVT)) return RET_EUNSUPPORTED;
  if (REV && C > 128) return RET_EUNSUPPORTED;
  const int BH = s.B * s.H;
  CUtensorMap mq, mk, mv, my;
  if (!make_map(&mq, q, DK, s.L, BH, C) || !make_map(&mk, k, DK, s.L, BH, C) ||
      !make_map(&mv, v, s.dv, s.L, BH, C) || !make_map(&my, y, s.dv, s.L, BH, C))
    return RET_ECUDA;
  static CwDecay dec;  // staged on the host; copied into the launch's parameters
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  fill_l2g(dec, gamma, s.H);

  const int smax = max_smem_optin();
  int ns = 0;
  if (C <= 128) {
    for (int n = kCW_MaxStages; n >= 1; --n)
      if ((int)cw_smem_plan(DK, C, n).total <= smax) { ns = n; break; }
    // the dk <= 128 kernel stages y in a V buffer while the next block's V
    // loads into another: two stages at least
    if (DK <= 128 && ns < 2) ns = 0;
  } else if (DK <= 128 && (int)cw_wide_smem_plan(DK, C).total <= smax) {
    ns = 1;  // blocks of 129..256 rows: one stage, two row halves
  }
  if (ns == 0) return RET_EUNSUPPORTED;
  CwSmem plan = cw_smem_plan(DK, C, ns);

  int n_seg = 1, seg_chunks = 0;
  plan_segments(s, C, &n_seg, &seg_chunks);
  if (force) n_seg = force->n_seg, seg_chunks = force->seg_chunks;
  if (reuse) n_seg = reuse->plan.n_seg, seg_chunks = reuse->plan.seg_chunks;
  while (!reuse && n_seg > 1 && (ws == nullptr || seg_workspace_bytes(s, n_seg) > ws_bytes)) {
    // not enough workspace for this split: fall back to fewer segments
    const int n_chunks = (s.L + C - 1) / C;
    int g = n_seg - 1;
    seg_chunks = (n_chunks + g - 1) / g;
    n_seg = (n_chunks + seg_chunks - 1) / seg_chunks;
  }
  if (n_seg <= 1) {
    if (reuse) return RET_EINVAL;
    n_seg = 1;
    seg_chunks = (s.L + C - 1) / C;
  }
  if (used) used->n_seg = n_seg, used->seg_chunks = seg_chunks;

  CwArgs a;
  a.B = s.B;
  a.H = s.H;
  a.L = s.L;
  a.dv = s.dv;
  a.C = C;
  a.seg_chunks = seg_chunks;
  a.n_seg = n_seg;
  a.nstages = ns;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.state_in = state_in;
  a.state_out = state_out;
  a.seg_state = reuse ? nullptr : static_cast<const float*>(ws);
  a.seg_tr = reuse ? reuse->src : nullptr;
  a.seg_tr_nseg = reuse ? reuse->n_src : 0;
  a.seg_tr_step = reuse ? reuse->step : 0;
  a.gn_eps = gn ? gn->eps : 0.f;
  a.gn_w = gn ? gn->weight : nullptr;
  a.gn_b = gn ? gn->bias : nullptr;
  a.lim = wait_limit();
  a.debug_drop_block = debug_drop_block();

  if (n_seg > 1 && !reuse) {
    // segment sums -> workspace slots 1..n_seg-1, then the scan fills every slot
    int ns2 = 0;
    const uint32_t per = (uint32_t)(DK / 64) * C * 128 + 2u * C * 128;
    for (int n = kCW_MaxStages; n >= 1; --n)
      if ((int)(n * per + kMiscBytes + kSmemAlign) <= smax) { ns2 = n; break; }
    CwArgs a2 = a;
    a2.nstages = ns2;
    a2.debug_drop_block = -1;
    const int smem2 = (int)(ns2 * per + kMiscBytes + kSmemAlign);
    if (cudaFuncSetAttribute(chunk_state_kernel<DK, REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) !=
        cudaSuccess)
      return RET_ECUDA;
    dim3 g2(s.dv / kCW_DVT, BH, n_seg - 1);
    chunk_state_kernel<DK, REV><<<g2, kCW_Threads, smem2, st>>>(mk, mv, a2, dec, static_cast<float*>(ws));
    if (launch_status() != RET_OK) return RET_ECUDA;
    // The scan and the main kernel are launched behind the kernel before them
    // (programmatic dependent launch): their prologues overlap its tail, and
    // each waits (griddep_wait) before it reads the segment states.
    const long long total = (long long)BH * DK * s.dv;
    const int blocks = (int)std::min<long long>((total + 255) / 256, 1LL << 20);  // one element per thread
    if (launch_after(state_scan_kernel<REV>, dim3(blocks), dim3(256), 0, st, state_in, static_cast<float*>(ws), BH,
                     s.H, DK * s.dv, n_seg, seg_chunks * C, s.L - (n_seg - 1) * seg_chunks * C, dec) != RET_OK)
      return RET_ECUDA;
  }
  const bool after = n_seg > 1 && !reuse;
  dim3 grid(s.dv / kCW_DVT, BH, n_seg);
  if constexpr (DK == 256) {
    // one stage; scores and cross-block term fused into one wide MMA
    const Cw256Smem p256 = cw256_smem_plan(C);
    if ((int)p256.total > smax) return RET_EUNSUPPORTED;
    a.nstages = 1;
    if (cudaFuncSetAttribute(chunkwise_tc256_kernel<REV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)p256.total) != cudaSuccess)
      return RET_ECUDA;
    if (after) return launch_after(chunkwise_tc256_kernel<REV>, grid, dim3(kCW_MainThreads), p256.total, st, mq, mk,
                                   mv, a, dec);
    chunkwise_tc256_kernel<REV><<<grid, kCW_MainThreads, p256.total, st>>>(mq, mk, mv, a, dec);
    return launch_status();
  } else {
    if (C > 128) {
      const CwWideSmem pw = cw_wide_smem_plan(DK, C);
      if (cudaFuncSetAttribute(chunkwise_wide_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)pw.total) != cudaSuccess)
        return RET_ECUDA;
      if (after) return launch_after(chunkwise_wide_kernel<DK>, grid, dim3(kCW_MainThreads), pw.total, st, mq, mk,
                                     mv, a, dec);
      chunkwise_wide_kernel<DK><<<grid, kCW_MainThreads, pw.total, st>>>(mq, mk, mv, a, dec);
      return launch_status();
    }
    // the normalising epilogue is its own instance, so the plain kernels keep
    // their register allocation
    auto* kern = gn ? chunkwise_tc_kernel<DK, false, true> : chunkwise_tc_kernel<DK, REV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.total) != cudaSuccess)
      return RET_ECUDA;
    if (after) return launch_after(kern, grid, dim3(kCW_MainThreads), plan.total, st, mq, mk, mv, my, a, dec);
    kern<<<grid, kCW_MainThreads, plan.total, st>>>(mq, mk, mv, my, a, dec);
    return launch_status();
  }
}

// Launch state_fold_kernel: out = fold of n parts (see state_fold.cuh).
ret_status launch_state_fold(const float* state_in, const float* parts, float* out, const ret_shape& s,
                             const float* gamma, int n, const int* lens, long long part_stride,
                             long long bh_stride, cudaStream_t st, bool after = false) {
  HeadLog2 hl;
  FoldLens fl;
  for (int h = 0; h < s.H; ++h) hl.l2g[h] = log2_gamma(gamma[h]);
  for (int h = s.H; h < RET_MAX_HEADS; ++h) hl.l2g[h] = 0.f;
  for (int i = 0; i < kFoldMaxParts; ++i) fl.len[i] = i < n ? lens[i] : 0;
  const long long BH = (long long)s.B * s.H;
  const long long total = BH * s.dk * s.dv;
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>((total + 255) / 256, 8LL * sm_count()));
  if (after) return launch_after(state_fold_kernel, dim3(grid), dim3(256), 0, st, state_in, parts, out, BH, s.H,
                                 s.dk * s.dv, n, part_stride, bh_stride, hl, fl);
  state_fold_kernel<<<grid, 256, 0, st>>>(state_in, parts, out, BH, s.H, s.dk * s.dv, n, part_stride, bh_stride,
                                          hl, fl);
  return launch_status();
}

// Plan of a state-only call.  Its result does not depend on the block length
// (every row of K is scaled by its own decay to the segment end, and the sums
// accumulate in fp32 across blocks), so it runs blocks of kStateC rows, short
// enough for two CTAs per SM with three stages each at dk = 256, and enough
// segments for about two CTAs per SM; fewer when the workspace (n_seg + 1
// states per (b, h)) is short.  Returns n_seg, 0 when even one segment does
// not fit.
constexpr int kStateC = 48;

int state_only_segments(const ret_shape& s, size_t ws_bytes, int* seg_chunks) {
  const size_t per = (size_t)s.B * s.H * s.dk * s.dv * sizeof(float);
  const int n_chunks = (s.L + kStateC - 1) / kStateC;
  const long long base = (long long)(s.dv / kCW_DVT) * s.B * s.H;  // CTAs per segment
  int n_seg = (int)std::max<long long>(1, (2LL * sm_count()) / base);
  n_seg = std::max(1, std::min({n_seg, std::max(1, n_chunks / 2), kFoldMaxParts}));
  while (n_seg > 1 && (size_t)(n_seg + 1) * per > ws_bytes) --n_seg;
  if ((size_t)(n_seg + 1) * per > ws_bytes) return 0;
  *seg_chunks = (n_chunks + n_seg - 1) / n_seg;
  return (n_chunks + *seg_chunks - 1) / *seg_chunks;
}

// State-only chunkwise pass on the tensor cores: chunk_state_kernel writes each
// segment's sum D_g to slot g + 1 of the workspace [BH][n_seg + 1][dk][dv], and
// the fold joins them with state_in.
template <int DK>
ret_status launch_chunk_state(const void* k, const void* v, const float* gamma, const float* state_in,
                              float* state_out, const ret_shape& s, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int BH = s.B * s.H, C = kStateC;
  int seg_chunks = 1;
  const int n_seg = state_only_segments(s, ws_bytes, &seg_chunks);
  if (n_seg == 0 || !ws) return RET_EINVAL;
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, DK, s.L, BH, C) || !make_map(&mv, v, s.dv, s.L, BH, C)) return RET_ECUDA;
  static CwDecay dec;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  fill_l2g(dec, gamma, s.H);
  const int smax = max_smem_optin();
  const uint32_t per = (uint32_t)(DK / 64) * C * 128 + 2u * C * 128;
  // as many stages as let two CTAs share an SM when there are more CTAs than
  // SMs (and two stages fit so), else as many as fit
  int ns = 0;
  const long long ctas = (long long)(s.dv / kCW_DVT) * BH * n_seg;
  int cap = kCW_MaxStages;
  if (ctas > sm_count() && 2 * (int)(2 * per + kMiscBytes + kSmemAlign) <= smax)
    while (cap > 2 && 2 * (int)(cap * per + kMiscBytes + kSmemAlign) > smax) --cap;
  for (int n = cap; n >= 1; --n)
    if ((int)(n * per + kMiscBytes + kSmemAlign) <= smax) { ns = n; break; }
  if (ns == 0) return RET_EUNSUPPORTED;
  CwArgs a{};
  a.B = s.B;
  a.H = s.H;
  a.L = s.L;
  a.dv = s.dv;
  a.C = C;
  a.seg_chunks = seg_chunks;
  a.n_seg = n_seg + 1;  // slot stride: slot 0 unused, segment g -> slot g + 1
  a.nstages = ns;
  a.lim = wait_limit();
  a.debug_drop_block = -1;
  const int smem = (int)(ns * per + kMiscBytes + kSmemAlign);
  if (cudaFuncSetAttribute(chunk_state_kernel<DK, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return RET_ECUDA;
  dim3 grid(s.dv / kCW_DVT, BH, n_seg);
  chunk_state_kernel<DK, false><<<grid, kCW_Threads, smem, st>>>(mk, mv, a, dec, static_cast<float*>(ws));
  if (launch_status() != RET_OK) return RET_ECUDA;
  int lens[kFoldMaxParts];
  for (int g = 0; g < n_seg; ++g) lens[g] = std::min(s.L, (g + 1) * seg_chunks * C) - g * seg_chunks * C;
  const long long dkdv = (long long)DK * s.dv;
  return launch_state_fold(state_in, static_cast<const float*>(ws) + dkdv, state_out, s, gamma, n_seg, lens, dkdv,
                           (long long)(n_seg + 1) * dkdv, st, /*after=*/true);
}

template <int DK, int DVT, bool REV>
ret_status launch_parallel_tc(const void* q, const void* k, const void* v, const float* gamma, void* y,
                              const ret_shape& s, cudaStream_t st) {
  const int BH = s.B * s.H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, DK, s.L, BH, 128) || !make_map(&mk, k, DK, s.L, BH, 128) ||
      !make_map(&mv, v, s.dv, s.L, BH, 128))
    return RET_ECUDA;
  static CwDecay dec;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  fill_l2g(dec, gamma, s.H);
  const int smax = max_smem_optin();
  int ns = 0;
  for (int n = kCW_MaxStages; n >= 1; --n)
    if ((int)pa_smem_plan(DK, DVT, n).total <= smax) { ns = n; break; }
  if (ns == 0) return RET_EUNSUPPORTED;
  const PaSmem plan = pa_smem_plan(DK, DVT, ns);
  PaArgs a;
  a.B = s.B;
  a.H = s.H;
  a.L = s.L;
  a.dv = s.dv;
  a.n_qt = (s.L + 127) / 128;
  a.nstages = ns;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.lim = wait_limit();
  if (cudaFuncSetAttribute(parallel_tc_kernel<DK, DVT, REV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)plan.total) != cudaSuccess)
    return RET_ECUDA;
  // blockIdx.y = y pairs query tiles n_qt-1-y and y (one tile when they meet)
  dim3 grid(s.dv / DVT, (a.n_qt + 1) / 2, BH);
  parallel_tc_kernel<DK, DVT, REV><<<grid, kPA_Threads, plan.total, st>>>(mq, mk, mv, a, dec);
  return launch_status();
}

template <typename T, int VEC>
void launch_groupnorm_vec(unsigned blocks, cudaStream_t st, const void* y, void* out, long long rows,
                          const ret_shape& s, float eps, const float* w, const float* b, const void* gate, int act) {
  auto yi = static_cast<const T*>(y);
  auto yo = static_cast<T*>(out);
  auto gi = static_cast<const T*>(gate);
  if (gate)
    launch_groupnorm_rows<T, VEC, true>(blocks, st, yi, yo, rows, s.H, s.L, s.dv, eps, w, b, gi, act);
  else
    launch_groupnorm_rows<T, VEC, false>(blocks, st, yi, yo, rows, s.H, s.L, s.dv, eps, w, b, gi, act);
}

ret_status launch_groupnorm(const void* y, void* out, float eps, const float* w, const float* b,
                            const ret_shape& s, ret_dtype dt, cudaStream_t st, const void* gate = nullptr,
                            int act = 0) {
  const long long rows = (long long)s.B * s.H * s.L;
  if (rows == 0) return RET_OK;
  const unsigned blocks = (unsigned)((rows + kGN_RowsPerBlock - 1) / kGN_RowsPerBlock);
  const bool vec = s.dv % 128 == 0;
  if (dt == RET_BF16) {
    if (s.dv % 256 == 0)
      launch_groupnorm_vec<__nv_bfloat16, 8>(blocks, st, y, out, rows, s, eps, w, b, gate, act);
    else if (vec)
      launch_groupnorm_vec<__nv_bfloat16, 4>(blocks, st, y, out, rows, s, eps, w, b, gate, act);
    else
      launch_groupnorm_vec<__nv_bfloat16, 1>(blocks, st, y, out, rows, s, eps, w, b, gate, act);
  } else {
    if (vec)
      launch_groupnorm_vec<float, 4>(blocks, st, y, out, rows, s, eps, w, b, gate, act);
    else
      launch_groupnorm_vec<float, 1>(blocks, st, y, out, rows, s, eps, w, b, gate, act);
  }
  return launch_status();
}

// Parallel form in either time direction: REV = false is retention_parallel,
// REV = true the anti-causal sum y_n = sum_{m>=n} gamma^(m-n) (q_n . k_m) v_m
// that the backward pass takes for dk and dv.
template <bool REV>
ret_status parallel_dir(const void* q, const void* k, const void* v, const float* gamma, void* y, ret_shape s,
                        ret_dtype dt, cudaStream_t st) {
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (s.L == 0) return RET_OK;
  if (!q || !k || !v || !y) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y)) return RET_EINVAL;
  if (dt == RET_F32) {
    if (s.dk > 256) return RET_EUNSUPPORTED;
    static HeadLog2 hl;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int h = 0; h < s.H; ++h) hl.l2g[h] = log2_gamma(gamma[h]);
    const int smem = (2 * kPF_Rows * (s.dk + 1) + kPF_Rows * kPF_Cols + kPF_Rows * 33) * 4;
    if (cudaFuncSetAttribute(parallel_f32_kernel<REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return RET_ECUDA;
    dim3 grid((s.dv + kPF_Cols - 1) / kPF_Cols, (s.L + kPF_Rows - 1) / kPF_Rows, s.B * s.H);
    parallel_f32_kernel<REV><<<grid, 256, smem, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                      static_cast<const float*>(v), static_cast<float*>(y), s.H,
                                                      s.L, s.dk, s.dv, hl);
    return launch_status();
  }
  if (dt != RET_BF16) return RET_EINVAL;
  if (!parallel_tc_shape_ok(s) || !device_is_sm100()) return RET_EUNSUPPORTED;
  const bool wide = s.dv % 128 == 0;  // 128-column dv slices, else 64
  switch (s.dk) {
    case 64: return wide ? launch_parallel_tc<64, 128, REV>(q, k, v, gamma, y, s, st)
                         : launch_parallel_tc<64, 64, REV>(q, k, v, gamma, y, s, st);
    case 128: return wide ? launch_parallel_tc<128, 128, REV>(q, k, v, gamma, y, s, st)
                          : launch_parallel_tc<128, 64, REV>(q, k, v, gamma, y, s, st);
    default: return wide ? launch_parallel_tc<256, 128, REV>(q, k, v, gamma, y, s, st)
                         : launch_parallel_tc<256, 64, REV>(q, k, v, gamma, y, s, st);
  }
}

// Chunkwise form in either time direction.  REV = false is retention_chunkwise.
// REV = true is the anti-causal sum, which the backward pass takes for dk and
// dv without reversing the sequence in memory:
//     y_n = sum_{m>=n} gamma^(m-n) (q_n . k_m) v_m + gamma^(L-n) q_n S_in,
// walked from the last block to the first, with state_in the state after the
// sequence and state_out = gamma^L S_in + sum_m gamma^m k_m^T v_m the state at
// its start (bf16: blocks of at most 128 rows).
template <bool REV>
ret_status chunkwise_dir(const void* q, const void* k, const void* v, const float* gamma, void* y,
                         const float* state_in, float* state_out, int chunk, ret_shape s, ret_dtype dt,
                         void* workspace, size_t workspace_bytes, cudaStream_t st, const SegPlan* force = nullptr,
                         SegPlan* used = nullptr, const SegReuse* reuse = nullptr, const GnParams* gn = nullptr) {
  if (used) used->n_seg = 0, used->seg_chunks = 0;  // no split unless the tensor-core path reports one
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (chunk < 1) return RET_EINVAL;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (s.L > 0 && (!q || !k || !v || !y)) return RET_EINVAL;
  if (s.L > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y))) return RET_EINVAL;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out))) return RET_EINVAL;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RET_EINVAL;
  if (dt == RET_F32) {
    if (chunk > kCF_MaxC || s.dk > 256) return RET_EUNSUPPORTED;
  } else {
    if (!tc_chunk_ok(chunk, s.dk)) return RET_EUNSUPPORTED;
    if (!tc_shape_ok(s)) return RET_EUNSUPPORTED;
    if (s.L > 0 && !device_is_sm100()) return RET_EUNSUPPORTED;
  }
  const size_t sbytes = (size_t)s.B * s.H * s.dk * s.dv * sizeof(float);
  if (s.L == 0) {  // nothing to compute: the state passes through
    if (!state_out) return RET_OK;
    cudaError_t e = state_in ? (state_in == state_out ? cudaSuccess
                                                      : cudaMemcpyAsync(state_out, state_in, sbytes,
                                                                        cudaMemcpyDeviceToDevice, st))
                             : cudaMemsetAsync(state_out, 0, sbytes, st);
    return e == cudaSuccess ? RET_OK : RET_ECUDA;
  }
  if (gn && (dt != RET_BF16 || s.dk > 128)) return RET_EUNSUPPORTED;
  if (dt == RET_F32) {
    static HeadLog2 hl;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int h = 0; h < s.H; ++h) hl.l2g[h] = log2_gamma(gamma[h]);
    const int smem = (s.dk * kCF_Cols + chunk * (chunk + 1) + chunk + 1) * 4;
    if (cudaFuncSetAttribute(chunkwise_f32_kernel<REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return RET_ECUDA;
    dim3 grid((s.dv + kCF_Cols - 1) / kCF_Cols, s.B * s.H);
    chunkwise_f32_kernel<REV><<<grid, 256, smem, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                  static_cast<const float*>(v), static_cast<float*>(y), state_in,
                                                  state_out, s.H, s.L, s.dk, s.dv, chunk, hl);
    return launch_status();
  }
  switch (s.dk) {
    case 64:
      return launch_chunkwise_tc<64, REV>(q, k, v, gamma, y, state_in, state_out, chunk, s, workspace,
                                          workspace_bytes, st, force, used, reuse, gn);
    case 128:
      return launch_chunkwise_tc<128, REV>(q, k, v, gamma, y, state_in, state_out, chunk, s, workspace,
                                           workspace_bytes, st, force, used, reuse, gn);
    default:
      if (reuse) return RET_EINVAL;
      return launch_chunkwise_tc<256, REV>(q, k, v, gamma, y, state_in, state_out, chunk, s, workspace,
                                           workspace_bytes, st, force, used, nullptr);
  }
}

// ---------------------------------------------------------------------------
// Host-buffer chunkwise (retention_chunkwise_host): the (b, h) rows are cut
// into groups of consecutive heads of one batch row; each group's copies in,
// kernels and copy out go to three streams ordered by events.

struct HostGroups {
  int heads;    // heads per group (the last group of a batch row may have fewer)
  int per_row;  // groups per batch row
};

HostGroups plan_host_groups(const ret_shape& s, int n_groups) {
  if (n_groups <= 0) n_groups = 8;
  const long long rows = (long long)s.B * s.H;
  int hpg = (int)std::min<long long>(s.H, std::max<long long>(1, (rows + n_groups - 1) / n_groups));
  HostGroups g;
  g.heads = hpg;
  g.per_row = (s.H + hpg - 1) / hpg;
  return g;
}

// Copy streams of one device, created on first use and kept for the process.
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
};

ret_status copy_streams(CopyStreams* out) {
  static std::mutex mu;
  static CopyStreams per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RET_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  CopyStreams& cs = per_dev[dev];
  if (!cs.h2d && cudaStreamCreateWithFlags(&cs.h2d, cudaStreamNonBlocking) != cudaSuccess) return RET_ECUDA;
  if (!cs.d2h && cudaStreamCreateWithFlags(&cs.d2h, cudaStreamNonBlocking) != cudaSuccess) return RET_ECUDA;
  *out = cs;
  return RET_OK;
}

// A pool of timing-free events per device, grown on demand and reused.  Calls
// on one device are serialised by the pool's lock while they enqueue, so the
// events of one call are not re-recorded by another before this call's waits
// are enqueued (a wait captures the event's state when it is enqueued).
struct EventPool {
  std::mutex mu;
  std::vector<cudaEvent_t> ev[64];
};

EventPool& event_pool() {
  static EventPool p;
  return p;
}

// ---------------------------------------------------------------------------
// Scratch for retention_chunkwise_static_ws: a fixed array in this library's
// device memory, for callers that cannot allocate.  Its size is the most
// sequence-split scratch that entry point accepts.  Every GPU that loads the
// library holds it until the process exits.
constexpr size_t kStaticWsBytes = (size_t)16 << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of g_static_ws for the current device.  The host-side name of
// a __device__ array is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
void* static_ws_address(ret_status* rc) {
  constexpr int kMaxDevices = 64;
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *rc = RET_ECUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) {
      *rc = RET_ECUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *rc = RET_OK;
  return addr[dev];
}

}  // namespace

extern "C" {

#ifdef RET_TRACE
// Trace builds only: route RET_TRACE_STAMP events to `buf` (device memory of
// n_ctas * blocks * events u64), or switch tracing off with buf = NULL.
RET_API int retention_debug_trace(void* buf, int blocks, int events) {
  unsigned long long* p = static_cast<unsigned long long*>(buf);
  if (cudaMemcpyToSymbol(g_trace_buf, &p, sizeof(p)) != cudaSuccess) return 1;
  if (cudaMemcpyToSymbol(g_trace_blocks, &blocks, sizeof(int)) != cudaSuccess) return 1;
  if (cudaMemcpyToSymbol(g_trace_events, &events, sizeof(int)) != cudaSuccess) return 1;
  return 0;
}
#endif

int retention_abi_version(void) { return 104; }

const char* retention_status_str(ret_status st) {
  switch (st) {
    case RET_OK: return "RET_OK";
    case RET_EINVAL: return "RET_EINVAL";
    case RET_EUNSUPPORTED: return "RET_EUNSUPPORTED";
    case RET_ECUDA: return "RET_ECUDA";
    case RET_ETIMEOUT: return "RET_ETIMEOUT";
    case RET_EBOUNDS: return "RET_EBOUNDS";
  }
  return "RET_UNKNOWN";
}

ret_status retention_get_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RET_ECUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_status, sizeof(int)) != cudaSuccess) return RET_ECUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return RET_ECUDA;
    return h == 5 ? RET_EBOUNDS : RET_ETIMEOUT;
  }
  return RET_OK;
}

#ifdef RET_BOUNDS_CHECK
// Bounds-checked builds only: the site number of the first failed index check
// since the last call (0: none), cleared by the call.
RET_API unsigned int retention_debug_bounds_site(void) {
  unsigned int site = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&site, g_bc_site, sizeof(site)) != cudaSuccess) return ~0u;
  cudaMemcpyToSymbol(g_bc_site, &zero, sizeof(zero));
  return site;
}
#endif

ret_status retention_recurrent_step(const void* q, const void* k, const void* v, const float* gamma,
                                    void* y, float* state, ret_shape s, ret_dtype dt, void* stream) {
  NvtxRange nvtx_range("retention_recurrent_step");
  ret_status rc = check_shape(s, false);
  if (rc != RET_OK) return rc;
  if (!q || !k || !v || !y || !state) return RET_EINVAL;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (s.dk > kDecodeMaxDk) return RET_EUNSUPPORTED;
  if (!aligned16(state)) return RET_EINVAL;
  static HeadGamma hg;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int h = 0; h < s.H; ++h) hg.g[h] = gamma[h];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid((s.dv + kDecodeCols - 1) / kDecodeCols, s.B * s.H);
  const bool vec = (s.dv % 4) == 0;
  if ((long long)grid.x * grid.y < 2LL * sm_count()) {
    // few heads: narrower column blocks, four times the CTAs
    const dim3 gn((s.dv + kDecodeNarrowCols - 1) / kDecodeNarrowCols, s.B * s.H);
    if (dt == RET_F32)
      recurrent_step_narrow_kernel<float><<<gn, kDecodeThreads, 0, st>>>(
          static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
          static_cast<float*>(y), state, s.H, s.dk, s.dv, hg);
    else
      recurrent_step_narrow_kernel<__nv_bfloat16><<<gn, kDecodeThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
          static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(y), state, s.H, s.dk, s.dv, hg);
    return launch_status();
  }
  if (dt == RET_F32) {
    auto* qf = static_cast<const float*>(q);
    auto* kf = static_cast<const float*>(k);
    auto* vf = static_cast<const float*>(v);
    auto* yf = static_cast<float*>(y);
    if (vec) recurrent_step_kernel<float, true><<<grid, kDecodeThreads, 0, st>>>(qf, kf, vf, yf, state, s.H, s.dk, s.dv, hg);
    else recurrent_step_kernel<float, false><<<grid, kDecodeThreads, 0, st>>>(qf, kf, vf, yf, state, s.H, s.dk, s.dv, hg);
  } else {
    auto* qb = static_cast<const __nv_bfloat16*>(q);
    auto* kb = static_cast<const __nv_bfloat16*>(k);
    auto* vb = static_cast<const __nv_bfloat16*>(v);
    auto* yb = static_cast<__nv_bfloat16*>(y);
    if (vec) recurrent_step_kernel<__nv_bfloat16, true><<<grid, kDecodeThreads, 0, st>>>(qb, kb, vb, yb, state, s.H, s.dk, s.dv, hg);
    else recurrent_step_kernel<__nv_bfloat16, false><<<grid, kDecodeThreads, 0, st>>>(qb, kb, vb, yb, state, s.H, s.dk, s.dv, hg);
  }
  return launch_status();
}

ret_status retention_parallel(const void* q, const void* k, const void* v, const float* gamma, void* y,
                              ret_shape s, ret_dtype dt, void* stream) {
  NvtxRange nvtx_range("retention_parallel");
  return parallel_dir<false>(q, k, v, gamma, y, s, dt, static_cast<cudaStream_t>(stream));
}

size_t retention_chunkwise_workspace_bytes(int chunk, ret_shape s, ret_dtype dt) {
  if (dt != RET_BF16 || !tc_chunk_ok(chunk, s.dk)) return 0;
  if (check_shape(s, true) != RET_OK || s.L < 1 || !tc_shape_ok(s)) return 0;
  int n_seg = 1, seg_chunks = 1;
  plan_segments(s, chunk, &n_seg, &seg_chunks);
  return seg_workspace_bytes(s, n_seg);
}

ret_status retention_chunkwise(const void* q, const void* k, const void* v, const float* gamma, void* y,
                               const float* state_in, float* state_out, int chunk, ret_shape s,
                               ret_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("retention_chunkwise");
  return chunkwise_dir<false>(q, k, v, gamma, y, state_in, state_out, chunk, s, dt, workspace, workspace_bytes,
                              static_cast<cudaStream_t>(stream));
}

size_t retention_chunkwise_state_workspace_bytes(int chunk, ret_shape s, ret_dtype dt) {
  if (check_shape(s, true) != RET_OK || chunk < 1 || dt != RET_BF16 || s.L == 0) return 0;
  if (!tc_chunk_ok(chunk, s.dk) || !tc_shape_ok(s)) return 0;
  int sc = 1;
  const int n_seg = state_only_segments(s, SIZE_MAX, &sc);
  return (size_t)(n_seg + 1) * s.B * s.H * s.dk * s.dv * sizeof(float);
}

ret_status retention_chunkwise_state(const void* k, const void* v, const float* gamma, const float* state_in,
                                     float* state_out, int chunk, ret_shape s, ret_dtype dt, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("retention_chunkwise_state");
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (chunk < 1) return RET_EINVAL;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (!state_out || !aligned16(state_out) || (state_in && !aligned16(state_in))) return RET_EINVAL;
  if (s.L > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return RET_EINVAL;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RET_EINVAL;
  if (dt == RET_F32) {
    if (chunk > kCF_MaxC || s.dk > 256) return RET_EUNSUPPORTED;
  } else {
    if (!tc_chunk_ok(chunk, s.dk) || !tc_shape_ok(s)) return RET_EUNSUPPORTED;
    if (s.L > 0 && !device_is_sm100()) return RET_EUNSUPPORTED;
    if (s.L > 0 && (!workspace || workspace_bytes < (size_t)2 * s.B * s.H * s.dk * s.dv * sizeof(float)))
      return RET_EINVAL;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.L == 0) {  // the state passes through
    const size_t sbytes = (size_t)s.B * s.H * s.dk * s.dv * sizeof(float);
    cudaError_t e = state_in ? (state_in == state_out ? cudaSuccess
                                                      : cudaMemcpyAsync(state_out, state_in, sbytes,
                                                                        cudaMemcpyDeviceToDevice, st))
                             : cudaMemsetAsync(state_out, 0, sbytes, st);
    return e == cudaSuccess ? RET_OK : RET_ECUDA;
  }
  if (dt == RET_F32) {  // the fp32 chunkwise kernel without its output (q unused)
    static HeadLog2 hl;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int h = 0; h < s.H; ++h) hl.l2g[h] = log2_gamma(gamma[h]);
    const int smem = (s.dk * kCF_Cols + chunk * (chunk + 1) + chunk + 1) * 4;
    if (cudaFuncSetAttribute(chunkwise_f32_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return RET_ECUDA;
    dim3 grid((s.dv + kCF_Cols - 1) / kCF_Cols, s.B * s.H);
    chunkwise_f32_kernel<false><<<grid, 256, smem, st>>>(static_cast<const float*>(k), static_cast<const float*>(k),
                                                  static_cast<const float*>(v), nullptr, state_in, state_out, s.H,
                                                  s.L, s.dk, s.dv, chunk, hl);
    return launch_status();
  }
  switch (s.dk) {
    case 64: return launch_chunk_state<64>(k, v, gamma, state_in, state_out, s, workspace, workspace_bytes, st);
    case 128: return launch_chunk_state<128>(k, v, gamma, state_in, state_out, s, workspace, workspace_bytes, st);
    default: return launch_chunk_state<256>(k, v, gamma, state_in, state_out, s, workspace, workspace_bytes, st);
  }
}

ret_status retention_state_fold(const float* parts, const int* lens, int n, const float* gamma,
                                const float* state_in, float* state_out, ret_shape s, void* stream) {
  NvtxRange nvtx_range("retention_state_fold");
  ret_status rc = check_shape(s, false);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (n < 0 || n > kFoldMaxParts || !state_out) return RET_EINVAL;
  if (n > 0 && (!parts || !lens)) return RET_EINVAL;
  for (int i = 0; i < n; ++i)
    if (lens[i] < 0) return RET_EINVAL;
  if ((parts && !aligned16(parts)) || !aligned16(state_out) || (state_in && !aligned16(state_in)))
    return RET_EINVAL;
  const long long per = (long long)s.B * s.H * s.dk * s.dv;
  if (n > 0) {  // state_out must not overlap the parts (state_in may be state_out)
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(parts), p1 = p0 + (uintptr_t)n * per * sizeof(float);
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(state_out), o1 = o0 + (uintptr_t)per * sizeof(float);
    if (o0 < p1 && p0 < o1) return RET_EINVAL;
  }
  return launch_state_fold(state_in, parts, state_out, s, gamma, n, lens, per, (long long)s.dk * s.dv,
                           static_cast<cudaStream_t>(stream));
}

// Chunkwise form with the sequence-split scratch taken from g_static_ws
// instead of a caller buffer (see the header for who needs this).
ret_status retention_chunkwise_static_ws(const void* q, const void* k, const void* v, const float* gamma,
                                         void* y, const float* state_in, float* state_out, int chunk,
                                         ret_shape s, ret_dtype dt, void* stream) {
  NvtxRange nvtx_range("retention_chunkwise_static_ws");
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (chunk < 1) return RET_EINVAL;
  // The address is looked up on every call (cached per device after the
  // first), so the first call on a device does the lookup whatever its shape.
  void* ws = static_ws_address(&rc);
  if (rc != RET_OK) return rc;
  const size_t need = retention_chunkwise_workspace_bytes(chunk, s, dt);
  if (need > kStaticWsBytes) return RET_EUNSUPPORTED;  // beyond the fixed scratch
  return retention_chunkwise(q, k, v, gamma, y, state_in, state_out, chunk, s, dt, need > 0 ? ws : nullptr,
                             need > 0 ? kStaticWsBytes : 0, stream);
}

size_t retention_chunkwise_host_workspace_bytes(int chunk, ret_shape s, ret_dtype dt, int n_groups) {
  if (check_shape(s, true) != RET_OK) return 0;
  const HostGroups g = plan_host_groups(s, n_groups);
  ret_shape gs = s;
  gs.B = 1;
  gs.H = g.heads;
  return retention_chunkwise_workspace_bytes(chunk, gs, dt);
}

ret_status retention_chunkwise_host(const void* q_host, const void* k_host, const void* v_host,
                                    const float* gamma, void* y_host, void* q_dev, void* k_dev, void* v_dev,
                                    void* y_dev, const float* state_in, float* state_out, int chunk,
                                    ret_shape s, ret_dtype dt, void* workspace, size_t workspace_bytes,
                                    int n_groups, void* stream) {
  NvtxRange nvtx_range("retention_chunkwise_host");
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (chunk < 1) return RET_EINVAL;
  if (s.L > 0 && (!q_host || !k_host || !v_host || !y_host || !q_dev || !k_dev || !v_dev || !y_dev))
    return RET_EINVAL;
  if (s.L == 0)  // nothing to copy: the state passes through as in retention_chunkwise
    return retention_chunkwise(q_dev, k_dev, v_dev, gamma, y_dev, state_in, state_out, chunk, s, dt,
                               workspace, workspace_bytes, stream);
  // Shape support and alignment are checked once for the whole call (every
  // group's pointers are the bases plus whole rows), so no group fails on them.
  if (dt == RET_F32 ? (chunk > kCF_MaxC || s.dk > 256)
                    : (!tc_chunk_ok(chunk, s.dk) || !tc_shape_ok(s) || !device_is_sm100()))
    return RET_EUNSUPPORTED;
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(y_dev) ||
      (state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)) ||
      (((size_t)s.L * s.dk * (dt == RET_BF16 ? 2 : 4)) & 15u) || (((size_t)s.L * s.dv * (dt == RET_BF16 ? 2 : 4)) & 15u) ||
      (((size_t)s.dk * s.dv * 4) & 15u))
    return RET_EINVAL;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CopyStreams cs;
  if ((rc = copy_streams(&cs)) != RET_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RET_ECUDA;

  const HostGroups g = plan_host_groups(s, n_groups);
  const int n_total = s.B * g.per_row;
  const size_t es = dt == RET_BF16 ? 2 : 4;
  const size_t qk_row = (size_t)s.L * s.dk * es, v_row = (size_t)s.L * s.dv * es;
  const size_t st_row = (size_t)s.dk * s.dv;

  EventPool& pool = event_pool();
  std::lock_guard<std::mutex> lock(pool.mu);
  std::vector<cudaEvent_t>& ev = pool.ev[dev];
  const size_t need = 2 * (size_t)n_total + 2;
  while (ev.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return RET_ECUDA;
    ev.push_back(e);
  }
  cudaEvent_t e_start = ev[0], e_done = ev[1];
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // everything after the work already on `stream`
  if (!ok(cudaEventRecord(e_start, st)) || !ok(cudaStreamWaitEvent(cs.h2d, e_start, 0)) ||
      !ok(cudaStreamWaitEvent(cs.d2h, e_start, 0)))
    return RET_ECUDA;
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* yh = static_cast<char*>(y_host);
  char* qd = static_cast<char*>(q_dev);
  char* kd = static_cast<char*>(k_dev);
  char* vd = static_cast<char*>(v_dev);
  char* yd = static_cast<char*>(y_dev);
  int gi = 0;
  for (int b = 0; b < s.B; ++b) {
    for (int h0 = 0; h0 < s.H; h0 += g.heads, ++gi) {
      const int nh = std::min(g.heads, s.H - h0);
      const size_t r0 = (size_t)b * s.H + h0;  // first (b, h) row of the group
      cudaEvent_t e_in = ev[2 + 2 * gi], e_out = ev[3 + 2 * gi];
      if (!ok(cudaMemcpyAsync(qd + r0 * qk_row, qh + r0 * qk_row, nh * qk_row, cudaMemcpyHostToDevice, cs.h2d)) ||
          !ok(cudaMemcpyAsync(kd + r0 * qk_row, kh + r0 * qk_row, nh * qk_row, cudaMemcpyHostToDevice, cs.h2d)) ||
          !ok(cudaMemcpyAsync(vd + r0 * v_row, vh + r0 * v_row, nh * v_row, cudaMemcpyHostToDevice, cs.h2d)) ||
          !ok(cudaEventRecord(e_in, cs.h2d)) || !ok(cudaStreamWaitEvent(st, e_in, 0)))
        return RET_ECUDA;
      ret_shape gs = s;
      gs.B = 1;
      gs.H = nh;
      rc = retention_chunkwise(qd + r0 * qk_row, kd + r0 * qk_row, vd + r0 * v_row, gamma + h0,
                               yd + r0 * v_row, state_in ? state_in + r0 * st_row : nullptr,
                               state_out ? state_out + r0 * st_row : nullptr, chunk, gs, dt, workspace,
                               workspace_bytes, stream);
      if (rc != RET_OK) return rc;
      if (!ok(cudaEventRecord(e_out, st)) || !ok(cudaStreamWaitEvent(cs.d2h, e_out, 0)) ||
          !ok(cudaMemcpyAsync(yh + r0 * v_row, yd + r0 * v_row, nh * v_row, cudaMemcpyDeviceToHost, cs.d2h)))
        return RET_ECUDA;
    }
  }
  // the call's work ends on `stream` once the last copy out is done
  if (!ok(cudaEventRecord(e_done, cs.d2h)) || !ok(cudaStreamWaitEvent(st, e_done, 0))) return RET_ECUDA;
  return RET_OK;
}

ret_status retention_groupnorm_gated(const void* y, const void* gate, void* out, float eps, const float* weight,
                                     const float* bias, int act, ret_shape s, ret_dtype dt, void* stream) {
  NvtxRange nvtx_range("retention_groupnorm_gated");
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (!(eps >= 0.f) || !std::isfinite(eps)) return RET_EINVAL;
  if (act < kGateNone || act > kGateSigmoid) return RET_EINVAL;
  if (s.L > 0 && (!y || !out)) return RET_EINVAL;
  if (s.dv > kGN_MaxDv) return RET_EUNSUPPORTED;
  const size_t es = dt == RET_BF16 ? 2 : 4;
  if (s.dv % 128 == 0 && (!aligned16(y) || !aligned16(out) || (gate && !aligned16(gate)))) return RET_EINVAL;
  if (s.L > 0 &&
      ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(gate)) % es))
    return RET_EINVAL;
  return launch_groupnorm(y, out, eps, weight, bias, s, dt, static_cast<cudaStream_t>(stream), gate, act);
}

ret_status retention_groupnorm(const void* y, void* out, float eps, const float* weight, const float* bias,
                               ret_shape s, ret_dtype dt, void* stream) {
  return retention_groupnorm_gated(y, nullptr, out, eps, weight, bias, kGateNone, s, dt, stream);
}

size_t retention_chunkwise_gn_workspace_bytes(int chunk, ret_shape s, ret_dtype dt) {
  return retention_chunkwise_workspace_bytes(chunk, s, dt);
}

ret_status retention_chunkwise_gn(const void* q, const void* k, const void* v, const float* gamma, void* y,
                                  const float* state_in, float* state_out, int chunk, ret_shape s, ret_dtype dt,
                                  float eps, const float* weight, const float* bias, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return retention_chunkwise_gn_gated(q, k, v, gamma, y, state_in, state_out, chunk, s, dt, eps, weight, bias,
                                      nullptr, RET_GATE_NONE, workspace, workspace_bytes, stream);
}

ret_status retention_chunkwise_gn_gated(const void* q, const void* k, const void* v, const float* gamma, void* y,
                                        const float* state_in, float* state_out, int chunk, ret_shape s,
                                        ret_dtype dt, float eps, const float* weight, const float* bias,
                                        const void* gate, int act, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  NvtxRange nvtx_range("retention_chunkwise_gn_gated");
  if (!(eps >= 0.f) || !std::isfinite(eps)) return RET_EINVAL;
  if (act < kGateNone || act > kGateSigmoid) return RET_EINVAL;
  if (s.dv > kGN_MaxDv) return RET_EUNSUPPORTED;
  if (gate && s.L > 0) {
    // y is normalised in place while the gate is read: the two must not share
    // a byte (an offset view of y would be read after rows of it were written)
    const size_t bytes = (size_t)s.B * s.H * s.L * s.dv * (dt == RET_BF16 ? 2 : 4);
    const uintptr_t g0 = reinterpret_cast<uintptr_t>(gate), y0 = reinterpret_cast<uintptr_t>(y);
    if (!aligned16(gate) || (g0 < y0 + bytes && y0 < g0 + bytes)) return RET_EINVAL;
  }
  // One dv slice per head (dv = 128), bf16, dk <= 128, blocks of at most 128
  // rows, no gate, weight and bias 16-byte aligned (read as float4): the
  // chunkwise kernel normalises each row before it stores y (one kernel).
  // Otherwise the normalisation (and the gate) run as a second kernel over y.
  if (!gate && (!weight || aligned16(weight)) && (!bias || aligned16(bias)) && dt == RET_BF16 && s.dv == kCW_DVT && s.dk <= 128 && chunk >= 16 && chunk <= 128 && s.L > 0 &&
      tc_chunk_ok(chunk, s.dk) && tc_shape_ok(s) && check_shape(s, true) == RET_OK) {
    const GnParams gn{eps, weight, bias};
    return chunkwise_dir<false>(q, k, v, gamma, y, state_in, state_out, chunk, s, dt, workspace, workspace_bytes,
                                static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, &gn);
  }
  ret_status rc = retention_chunkwise(q, k, v, gamma, y, state_in, state_out, chunk, s, dt, workspace,
                                      workspace_bytes, stream);
  if (rc != RET_OK || s.L == 0) return rc;
  return retention_groupnorm_gated(y, gate, y, eps, weight, bias, act, s, dt, stream);
}

size_t retention_parallel_backward_workspace_bytes(ret_shape s, ret_dtype dt) {
  (void)s;
  (void)dt;
  return 0;  // the anti-causal sums read the inputs in place: no scratch
}

ret_status retention_parallel_backward(const void* q, const void* k, const void* v, const float* gamma,
                                       const void* dy, void* dq, void* dk, void* dv, ret_shape s, ret_dtype dt,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("retention_parallel_backward");
  (void)workspace;
  (void)workspace_bytes;
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (s.L == 0) return RET_OK;
  if (!q || !k || !v || !dy || !dq || !dk || !dv) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return RET_EINVAL;
  // the three sums take (dy, v, k), (v, dy, q) and (k, q, dy): both dk and dv
  // play the role of the key width
  if (dt == RET_BF16) {
    const ret_shape a{s.B, s.H, s.L, s.dv, s.dk}, b{s.B, s.H, s.L, s.dk, s.dv};
    if (!parallel_tc_shape_ok(a) || !parallel_tc_shape_ok(b) || !device_is_sm100()) return RET_EUNSUPPORTED;
  } else if (s.dk > 256 || s.dv > 256) {
    return RET_EUNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const ret_shape swapped{s.B, s.H, s.L, s.dv, s.dk};  // key width dv, value width dk
  // dq_n = sum_{m<=n} gamma^(n-m) (dy_n . v_m) k_m        (causal)
  if ((rc = parallel_dir<false>(dy, v, k, gamma, dq, swapped, dt, st)) != RET_OK) return rc;
  // dk_m = sum_{n>=m} gamma^(n-m) (v_m . dy_n) q_n        (anti-causal)
  if ((rc = parallel_dir<true>(v, dy, q, gamma, dk, swapped, dt, st)) != RET_OK) return rc;
  // dv_m = sum_{n>=m} gamma^(n-m) (k_m . q_n) dy_n        (anti-causal)
  return parallel_dir<true>(k, q, dy, gamma, dv, s, dt, st);
}

// Chunkwise variant: the same three retention sums through the chunkwise form,
// dq causal and dk, dv anti-causal (chunkwise_dir<true>), so nothing is
// reversed in memory; the workspace holds the sequence-split scratch of the
// largest of the three calls and, with a carried state, three fp32 states.
// One fp32 [B][H][dk][dv] state, rounded up to 256 bytes.
size_t state_region_bytes(const ret_shape& s) {
  return ((size_t)s.B * s.H * s.dk * s.dv * sizeof(float) + 255) & ~size_t(255);
}

// Block length of the two anti-causal sums: the anti-causal kernels take
// blocks of at most 128 rows (the result does not depend on it beyond
// rounding).
int rev_chunk(int chunk) { return std::min(chunk, 128); }

size_t chunkwise_backward_split_ws(int chunk, const ret_shape& s, ret_dtype dt) {
  const ret_shape swapped{s.B, s.H, s.L, s.dv, s.dk};
  const int cr = rev_chunk(chunk);
  return std::max({retention_chunkwise_workspace_bytes(chunk, swapped, dt),
                   retention_chunkwise_workspace_bytes(cr, swapped, dt),
                   retention_chunkwise_workspace_bytes(cr, s, dt)});
}

size_t retention_chunkwise_backward_workspace_bytes(int chunk, ret_shape s, ret_dtype dt) {
  if (check_shape(s, true) != RET_OK || (dt != RET_F32 && dt != RET_BF16)) return 0;
  return chunkwise_backward_split_ws(chunk, s, dt);
}

size_t retention_chunkwise_backward_state_workspace_bytes(int chunk, ret_shape s, ret_dtype dt) {
  if (check_shape(s, true) != RET_OK || (dt != RET_F32 && dt != RET_BF16)) return 0;
  return chunkwise_backward_split_ws(chunk, s, dt) + 3 * state_region_bytes(s);
}

ret_status retention_chunkwise_backward(const void* q, const void* k, const void* v, const float* gamma,
                                        const void* dy, void* dq, void* dk, void* dv, int chunk, ret_shape s,
                                        ret_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
  return retention_chunkwise_backward_state(q, k, v, gamma, dy, nullptr, nullptr, dq, dk, dv, nullptr, chunk, s, dt,
                                            workspace, workspace_bytes, stream);
}

ret_status retention_chunkwise_backward_state(const void* q, const void* k, const void* v, const float* gamma,
                                              const void* dy, const float* state_in, const float* dstate_out,
                                              void* dq, void* dk, void* dv, float* dstate_in, int chunk,
                                              ret_shape s, ret_dtype dt, void* workspace, size_t workspace_bytes,
                                              void* stream) {
  NvtxRange nvtx_range("retention_chunkwise_backward_state");
  ret_status rc = check_shape(s, true);
  if (rc != RET_OK) return rc;
  if ((rc = check_gamma(gamma, s.H)) != RET_OK) return rc;
  if (dt != RET_F32 && dt != RET_BF16) return RET_EINVAL;
  if (chunk < 1) return RET_EINVAL;
  const bool carried = state_in || dstate_out || dstate_in;
  if ((state_in && !aligned16(state_in)) || (dstate_out && !aligned16(dstate_out)) ||
      (dstate_in && !aligned16(dstate_in)))
    return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t sbytes = (size_t)s.B * s.H * s.dk * s.dv * sizeof(float);
  if (s.L == 0) {  // S_out = S0: dS0 = dS_out
    if (!dstate_in) return RET_OK;
    const cudaError_t e = dstate_out ? (dstate_out == dstate_in ? cudaSuccess
                                                                 : cudaMemcpyAsync(dstate_in, dstate_out, sbytes,
                                                                                   cudaMemcpyDeviceToDevice, st))
                                     : cudaMemsetAsync(dstate_in, 0, sbytes, st);
    return e == cudaSuccess ? RET_OK : RET_ECUDA;
  }
  if (!q || !k || !v || !dy || !dq || !dk || !dv) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return RET_EINVAL;
  const ret_shape swapped{s.B, s.H, s.L, s.dv, s.dk};  // key width dv, value width dk
  if (dt == RET_BF16) {
    if (!tc_shape_ok(s) || !tc_shape_ok(swapped) || !tc_chunk_ok(chunk, s.dk) || !tc_chunk_ok(chunk, s.dv) ||
        !device_is_sm100())
      return RET_EUNSUPPORTED;
  } else if (s.dk > 256 || s.dv > 256 || chunk > kCF_MaxC) {
    return RET_EUNSUPPORTED;
  }
  const size_t split = chunkwise_backward_split_ws(chunk, s, dt);
  const size_t sreg = carried ? state_region_bytes(s) : 0;
  if (split + 3 * sreg > 0 &&
      (!workspace || workspace_bytes < split + 3 * sreg || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
    return RET_EINVAL;
  char* w = static_cast<char*>(workspace);
  void* sw = split ? w : nullptr;
  // initial states of the three sums: S0^T, (dS_out / gamma)^T, dS_out / gamma;
  // the x2 region later takes the dv sum's state_out
  float* s0t = carried ? reinterpret_cast<float*>(w + split) : nullptr;
  float* x2 = carried ? reinterpret_cast<float*>(w + split + sreg) : nullptr;
  float* x3 = carried ? reinterpret_cast<float*>(w + split + 2 * sreg) : nullptr;
  const long long BH = (long long)s.B * s.H;
  HeadGamma hg, gl;
  bool any_small = false;
  for (int h = 0; h < s.H; ++h) {
    hg.g[h] = gamma[h];
    const bool small = !(gamma[h] >= kBwdMinGamma);
    gl.g[h] = small ? (float)std::pow((double)gamma[h], (double)s.L) : 0.f;
    any_small |= small;
  }
  for (int h = s.H; h < RET_MAX_HEADS; ++h) hg.g[h] = gl.g[h] = 0.f;
  if (state_in || dstate_out) {
    dim3 grid((s.dv + 31) / 32, (s.dk + 31) / 32, (unsigned)BH);
    bwd_state_prep_kernel<<<grid, dim3(32, 8), 0, st>>>(state_in, dstate_out, s0t, x2, x3, s.H, s.dk, s.dv, hg);
    if ((rc = launch_status()) != RET_OK) return rc;
  }
  const int cr = rev_chunk(chunk);
  // dq_n = sum_{m<=n} gamma^(n-m) (dy_n . v_m) k_m + gamma^(n+1) dy_n S0^T:  causal, state_in S0^T
  if ((rc = chunkwise_dir<false>(dy, v, k, gamma, dq, state_in ? s0t : nullptr, nullptr, chunk, swapped, dt, sw,
                                 split, st)) != RET_OK)
    return rc;
  // The two anti-causal sums carry transposed states (sum_n dy_n^T q_n and
  // sum_n q_n^T dy_n, from (dS_out / gamma)^T and dS_out / gamma).  When both
  // are split into segments, the dk sum runs with segments `step` times
  // shorter than the dv sum's, and the dv sum starts each segment from the
  // transpose of the dk sum's scanned state at the same token, with no
  // segment-sum pass of its own.
  SegPlan p3{}, p2{}, p2_used{};
  int step = 0;
  if (dt == RET_BF16 && s.dk <= 128) {
    plan_segments(s, cr, &p3.n_seg, &p3.seg_chunks);
    plan_segments(swapped, cr, &p2.n_seg, &p2.seg_chunks);
    if (p3.n_seg > 1 && p2.n_seg >= p3.n_seg) {
      for (step = p2.n_seg / p3.n_seg; step > 1 && p3.seg_chunks % step != 0; --step) {
      }
      const int n_chunks = (s.L + cr - 1) / cr;
      p2.seg_chunks = p3.seg_chunks / step;
      p2.n_seg = (n_chunks + p2.seg_chunks - 1) / p2.seg_chunks;
      if (p2.n_seg <= 1) step = 0;
    }
  }
  // dk_m = sum_{n>=m} gamma^(n-m) (v_m . dy_n) q_n + gamma^(L-1-m) v_m dS_out^T:  anti-causal, state_in x2
  if ((rc = chunkwise_dir<true>(v, dy, q, gamma, dk, dstate_out ? x2 : nullptr, nullptr, cr, swapped, dt, sw, split,
                                st, step ? &p2 : nullptr, &p2_used)) != RET_OK)
    return rc;
  const bool reuse_ok = step > 0 && p2_used.n_seg == p2.n_seg && p2_used.seg_chunks == p2.seg_chunks;
  const SegReuse reuse{static_cast<const float*>(sw), p2.n_seg, step, p3};
  // dv_m = sum_{n>=m} gamma^(n-m) (k_m . q_n) dy_n + gamma^(L-1-m) k_m dS_out:  anti-causal, state_in x3;
  // its state_out T = sum_n gamma^n q_n^T dy_n + gamma^(L-1) dS_out goes to x2 (dS0 = gamma T)
  if ((rc = chunkwise_dir<true>(k, q, dy, gamma, dv, dstate_out ? x3 : nullptr, dstate_in ? x2 : nullptr, cr, s, dt,
                                sw, split, st, nullptr, nullptr, reuse_ok ? &reuse : nullptr)) != RET_OK)
    return rc;
  if (dstate_out && any_small) {
    if (dt == RET_BF16)
      bwd_last_token_kernel<__nv_bfloat16><<<(unsigned)BH, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), dstate_out,
          static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), s.H, s.L, s.dk, s.dv, hg);
    else
      bwd_last_token_kernel<float><<<(unsigned)BH, 256, 0, st>>>(static_cast<const float*>(k),
                                                                 static_cast<const float*>(v), dstate_out,
                                                                 static_cast<float*>(dk), static_cast<float*>(dv),
                                                                 s.H, s.L, s.dk, s.dv, hg);
    if ((rc = launch_status()) != RET_OK) return rc;
  }
  if (dstate_in) {
    const long long total = BH * s.dk * s.dv;
    const unsigned grid = (unsigned)std::min<long long>((total + 255) / 256, 8LL * sm_count());
    bwd_finish_state_kernel<<<grid, 256, 0, st>>>(x2, dstate_out, dstate_in, BH, s.H, s.dk * s.dv, hg, gl);
    if ((rc = launch_status()) != RET_OK) return rc;
  }
  return RET_OK;
}

}  // extern "C"
