// C ABI entry points: argument checks, then the launchers of the kernel files.
#include <cmath>
#include <mutex>

#include "host.hpp"

namespace samba {

static thread_local std::string g_last_error;

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SAMBA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return SAMBA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
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

int encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle,
                 const char* what) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return fail(SAMBA_ERR_CUDA, "%s: cuTensorMapEncodeTiled is not available from the driver", what);
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAMBA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
  return SAMBA_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

static bool dtype_ok(int dt) { return dt == SAMBA_F32 || dt == SAMBA_BF16; }

}  // namespace samba

using namespace samba;

extern "C" {

int samba_version(void) { return 100; }

const char* samba_last_error(void) { return g_last_error.c_str(); }

int samba_get_status(samba_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int codes[5] = {take_status_scan(s), take_status_swa(s), take_status_misc(s), take_status_gemm(s),
                  take_status_swa_bwd(s)};
  for (int c : codes)
    if (c == SAMBA_ERR_CUDA) return fail(SAMBA_ERR_CUDA, "samba_get_status: %s", cudaGetErrorString(cudaGetLastError()));
  for (int c : codes)
    if (c != 0) return fail(c, "a kernel gave up a device-side wait");
  return SAMBA_OK;
}

int samba_selftest_wait_timeout(samba_stream_t stream) {
  return launch_selftest_wait(reinterpret_cast<cudaStream_t>(stream));
}

int samba_selftest_check(samba_stream_t stream) {
  return launch_selftest_check(reinterpret_cast<cudaStream_t>(stream));
}

int samba_conv1d_fwd(const void* x, int x_dtype, const float* w, const float* bias, const float* conv_state_in,
                     void* u, int u_dtype, float* conv_state_out, int64_t batch, int64_t seqlen, int64_t dim,
                     int dconv, int silu, samba_stream_t stream) {
  if (!x || !w || !u) return fail(SAMBA_ERR_INVALID_ARG, "samba_conv1d_fwd: x, w and u are required");
  if (batch < 1 || seqlen < 1 || dim < 1) return fail(SAMBA_ERR_INVALID_ARG, "samba_conv1d_fwd: bad shape");
  if (dconv < 2 || dconv > 4) return fail(SAMBA_ERR_UNSUPPORTED, "samba_conv1d_fwd: dconv must be 2..4");
  if (!dtype_ok(x_dtype) || !dtype_ok(u_dtype)) return fail(SAMBA_ERR_UNSUPPORTED, "samba_conv1d_fwd: dtype");
  if (seqlen > 1 && conv_state_in && conv_state_in == conv_state_out)
    return fail(SAMBA_ERR_INVALID_ARG, "samba_conv1d_fwd: conv_state_out may alias conv_state_in only for L = 1");
  if (!aligned16(x) || !aligned16(u)) return fail(SAMBA_ERR_INVALID_ARG, "samba_conv1d_fwd: misaligned pointer");
  return launch_conv1d(x, x_dtype, w, bias, conv_state_in, u, u_dtype, conv_state_out, batch, seqlen, dim, dconv,
                       silu, reinterpret_cast<cudaStream_t>(stream));
}

static int check_scan(const samba_scan_args* a, const char* who) {
  if (!a) return fail(SAMBA_ERR_INVALID_ARG, "%s: null args", who);
  if (!a->x || !a->delta || !a->A || !a->Bm || !a->Cm || !a->y)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: x, delta, A, Bm, Cm and y are required", who);
  if (a->batch < 1 || a->seqlen < 1 || a->dim < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (a->dim % 8 != 0) return fail(SAMBA_ERR_INVALID_ARG, "%s: dim must be a multiple of 8", who);
  if (a->seqlen > (int64_t(1) << 31) - 1024 || a->batch > 65535)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: seqlen or batch too large", who);
  if (a->dstate != 4 && a->dstate != 8 && a->dstate != 16)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: dstate must be 4, 8 or 16", who);
  if (a->dconv < 2 || a->dconv > 4) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dconv must be 2..4", who);
  if (!dtype_ok(a->x_dtype) || !dtype_ok(a->y_dtype) || (a->z && !dtype_ok(a->z_dtype)))
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: dtype must be SAMBA_F32 or SAMBA_BF16", who);
  if ((a->flags & SAMBA_SCAN_FUSE_CONV) && !a->conv_w)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: FUSE_CONV needs conv_w", who);
  if (a->flags & ~7u) return fail(SAMBA_ERR_INVALID_ARG, "%s: unknown flag bits", who);
  const void* ptrs[] = {a->x, a->z, a->delta, a->Bm, a->Cm, a->y, a->h_ckpt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  return SAMBA_OK;
}

static int check_swa(const samba_swa_args* a, const char* who) {
  if (!a) return fail(SAMBA_ERR_INVALID_ARG, "%s: null args", who);
  if (!a->q || !a->k || !a->v || !a->o) return fail(SAMBA_ERR_INVALID_ARG, "%s: q, k, v and o are required", who);
  if (a->batch < 1 || a->seqlen < 1 || a->window < 1 || a->heads_q < 1 || a->heads_kv < 1)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (a->heads_q % a->heads_kv != 0) return fail(SAMBA_ERR_INVALID_ARG, "%s: heads_q %% heads_kv != 0", who);
  const int group = a->heads_q / a->heads_kv;
  if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: heads_q / heads_kv must be 1, 2, 4, 8 or 16", who);
  if (a->head_dim != 16 && a->head_dim != 32 && a->head_dim != 64)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: head_dim must be 16, 32 or 64", who);
  if (a->seqlen > (int64_t(1) << 30) || a->batch > 65535)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: seqlen or batch too large", who);
  const void* ptrs[] = {a->q, a->k, a->v, a->o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  return SAMBA_OK;
}

size_t samba_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t dim, int32_t dstate) {
  if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1) return 0;
  return scan_bwd_workspace(batch, seqlen, dim, dstate);
}

static int check_scan_bwd(const samba_scan_bwd_args* a, const char* who) {
  if (!a) return fail(SAMBA_ERR_INVALID_ARG, "%s: null args", who);
  // the forward's checks on the shared fields
  samba_scan_args f = {};
  f.x = a->x;
  f.z = a->z;
  f.delta = a->delta;
  f.A = a->A;
  f.Bm = a->Bm;
  f.Cm = a->Cm;
  f.Dskip = a->Dskip;
  f.conv_w = a->conv_w;
  f.conv_b = a->conv_b;
  f.y = const_cast<void*>(a->dy);  // read only: checked like the forward output
  f.batch = a->batch;
  f.seqlen = a->seqlen;
  f.dim = a->dim;
  f.dstate = a->dstate;
  f.dconv = a->dconv;
  f.x_dtype = a->x_dtype;
  f.z_dtype = a->z_dtype;
  f.y_dtype = a->y_dtype;
  f.flags = a->flags;
  int rc = check_scan(&f, who);
  if (rc != SAMBA_OK) return rc;
  if (a->z && a->z_dtype != a->x_dtype) return fail(SAMBA_ERR_UNSUPPORTED, "%s: z dtype must equal x dtype", who);
  if (!a->dx || !a->ddelta || !a->dA || !a->dB || !a->dC)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: dy, dx, ddelta, dA, dB and dC are required", who);
  if ((a->z && !a->dz) || (a->Dskip && !a->dD))
    return fail(SAMBA_ERR_INVALID_ARG, "%s: dz is required with z and dD with Dskip", who);
  const bool fuse = (a->flags & SAMBA_SCAN_FUSE_CONV) != 0;
  if (fuse && (!a->dconv_w || (a->conv_b && !a->dconv_b)))
    return fail(SAMBA_ERR_INVALID_ARG, "%s: dconv_w (and dconv_b with conv_b) are required with FUSE_CONV", who);
  const void* ptrs[] = {a->dx, a->dz, a->ddelta, a->dB, a->dC, a->workspace, a->ckpt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  const size_t need = scan_bwd_workspace(a->batch, a->seqlen, a->dim, a->dstate);
  if (!a->workspace || need == SIZE_MAX || a->workspace_bytes < need)
    return fail(SAMBA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", who, need);
  return SAMBA_OK;
}

int samba_selective_scan_bwd(const samba_scan_bwd_args* a, samba_stream_t stream) {
  const int rc = check_scan_bwd(a, "samba_selective_scan_bwd");
  if (rc != SAMBA_OK) return rc;
  return launch_scan_bwd(*a, reinterpret_cast<cudaStream_t>(stream));
}

size_t samba_swa_bwd_workspace_size(int64_t batch, int64_t seqlen, int32_t heads_q) {
  if (batch < 1 || seqlen < 1 || heads_q < 1) return 0;
  return swa_bwd_workspace(batch, seqlen, heads_q);
}

static int check_swa_bwd(const samba_swa_bwd_args* a, const char* who) {
  if (!a) return fail(SAMBA_ERR_INVALID_ARG, "%s: null args", who);
  samba_swa_args f = {};
  f.q = a->q;
  f.k = a->k;
  f.v = a->v;
  f.o = const_cast<void*>(a->o);  // read only: checked like the forward output
  f.batch = a->batch;
  f.seqlen = a->seqlen;
  f.window = a->window;
  f.heads_q = a->heads_q;
  f.heads_kv = a->heads_kv;
  f.head_dim = a->head_dim;
  f.scale = a->scale;
  int rc = check_swa(&f, who);
  if (rc != SAMBA_OK) return rc;
  if (!a->lse || !a->dO || !a->dq || !a->dk || !a->dv)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: o, lse, dO, dq, dk and dv are required", who);
  const void* ptrs[] = {a->lse, a->dO, a->dq, a->dk, a->dv, a->workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  const size_t need = swa_bwd_workspace(a->batch, a->seqlen, a->heads_q);
  if (!a->workspace || need == SIZE_MAX || a->workspace_bytes < need)
    return fail(SAMBA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", who, need);
  return SAMBA_OK;
}

int samba_swa_bwd(const samba_swa_bwd_args* a, samba_stream_t stream) {
  const int rc = check_swa_bwd(a, "samba_swa_bwd");
  if (rc != SAMBA_OK) return rc;
  return launch_swa_bwd(*a, reinterpret_cast<cudaStream_t>(stream));
}

int samba_mixer_bwd(const samba_scan_bwd_args* scan, const samba_swa_bwd_args* swa, samba_stream_t stream,
                    samba_stream_t aux) {
  const char* who = "samba_mixer_bwd";
  int rc = check_scan_bwd(scan, who);
  if (rc != SAMBA_OK) return rc;
  rc = check_swa_bwd(swa, who);
  if (rc != SAMBA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t a = reinterpret_cast<cudaStream_t>(aux);
  if (!a) {
    rc = launch_scan_bwd(*scan, s);
    if (rc != SAMBA_OK) return rc;
    return launch_swa_bwd(*swa, s);
  }
  // The scan's backward goes first on `stream`; the attention's, forked onto
  // `aux`, takes the SMs the scan leaves free and is joined back, so that the
  // call as a whole stays ordered on `stream`.
  cudaEvent_t fork = nullptr, join = nullptr;
  if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess)
    return fail(SAMBA_ERR_CUDA, "%s: event creation failed", who);
  if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(fork);
    return fail(SAMBA_ERR_CUDA, "%s: event creation failed", who);
  }
  if (cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(a, fork, 0) != cudaSuccess) {
    rc = fail(SAMBA_ERR_CUDA, "%s: cannot fork the aux stream", who);
  } else {
    rc = launch_scan_bwd(*scan, s);
    // After a failed scan launch the attention is not started; the join below
    // still orders `stream` after whatever reached `aux`.
    if (rc == SAMBA_OK) rc = launch_swa_bwd(*swa, a);
    if ((cudaEventRecord(join, a) != cudaSuccess || cudaStreamWaitEvent(s, join, 0) != cudaSuccess) &&
        rc == SAMBA_OK)
      rc = fail(SAMBA_ERR_CUDA, "%s: cannot join the aux stream", who);
  }
  cudaEventDestroy(fork);
  cudaEventDestroy(join);
  return rc;
}

int samba_gemm(const samba_gemm_args* a, samba_stream_t stream) {
  const char* who = "samba_gemm";
  if (!a || !a->A || !a->B) return fail(SAMBA_ERR_INVALID_ARG, "%s: A and B are required", who);
  if (a->M < 1 || a->N < 1 || a->K < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (a->M > int64_t(65535) * 128 || a->N > INT32_MAX || a->K > INT32_MAX)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: M, N or K too large", who);
  if (a->lda < a->K || a->ldb < a->K || a->lda % 8 || a->ldb % 8)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: lda and ldb must be >= K and multiples of 8", who);
  if (!aligned16(a->A) || !aligned16(a->B)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned operand", who);
  if (a->nout < 1 || a->nout > 3) return fail(SAMBA_ERR_UNSUPPORTED, "%s: nout must be 1..3", who);
  for (int o = 0; o < a->nout; ++o) {
    const samba_gemm_out& out = a->out[o];
    if (!out.ptr) return fail(SAMBA_ERR_INVALID_ARG, "%s: output %d is NULL", who, o);
    if (!dtype_ok(out.dtype)) return fail(SAMBA_ERR_UNSUPPORTED, "%s: output %d dtype", who, o);
    if (out.col0 < 0 || out.col1 <= out.col0 || out.col1 > a->N)
      return fail(SAMBA_ERR_INVALID_ARG, "%s: output %d column range", who, o);
    if (out.ld < out.col1 - out.col0) return fail(SAMBA_ERR_INVALID_ARG, "%s: output %d row stride", who, o);
  }
  if (a->workspace && !aligned16(a->workspace)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned workspace", who);
  return launch_gemm(*a, reinterpret_cast<cudaStream_t>(stream));
}

size_t samba_gemm_workspace_size(int64_t M, int64_t N) { return gemm_workspace_size(M, N); }

int samba_selective_scan_fwd(const samba_scan_args* args, samba_stream_t stream) {
  int rc = check_scan(args, "samba_selective_scan_fwd");
  if (rc != SAMBA_OK) return rc;
  return launch_scan(*args, reinterpret_cast<cudaStream_t>(stream));
}

int samba_swa_fwd(const samba_swa_args* args, samba_stream_t stream) {
  int rc = check_swa(args, "samba_swa_fwd");
  if (rc != SAMBA_OK) return rc;
  return launch_swa(*args, reinterpret_cast<cudaStream_t>(stream));
}

int samba_mixer_prefill(const samba_scan_args* scan, const samba_swa_args* swa, samba_stream_t stream,
                        samba_stream_t aux) {
  int rc = check_scan(scan, "samba_mixer_prefill");
  if (rc != SAMBA_OK) return rc;
  rc = check_swa(swa, "samba_mixer_prefill");
  if (rc != SAMBA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t a = reinterpret_cast<cudaStream_t>(aux);
  if (!a) {
    rc = launch_swa(*swa, s);
    if (rc != SAMBA_OK) return rc;
    return launch_scan(*scan, s);
  }
  // Fork `aux` from `stream`, run the attention there and the scan on
  // `stream`, then join `aux` back, so that the call as a whole stays ordered
  // on `stream`.  The events are created per call and released at once (a
  // recorded event may be destroyed while its work is pending).
  cudaEvent_t fork = nullptr, join = nullptr;
  if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess)
    return fail(SAMBA_ERR_CUDA, "samba_mixer_prefill: event creation failed");
  if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(fork);
    return fail(SAMBA_ERR_CUDA, "samba_mixer_prefill: event creation failed");
  }
  if (cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(a, fork, 0) != cudaSuccess) {
    rc = fail(SAMBA_ERR_CUDA, "samba_mixer_prefill: cannot fork the aux stream");
  } else {
    rc = launch_swa(*swa, a);
    // After a failed attention launch the scan is not started; the join below
    // still orders `stream` after whatever reached `aux`.
    if (rc == SAMBA_OK) rc = launch_scan(*scan, s);
    if ((cudaEventRecord(join, a) != cudaSuccess || cudaStreamWaitEvent(s, join, 0) != cudaSuccess) &&
        rc == SAMBA_OK)
      rc = fail(SAMBA_ERR_CUDA, "samba_mixer_prefill: cannot join the aux stream");
  }
  cudaEventDestroy(fork);
  cudaEventDestroy(join);
  return rc;
}

int samba_scan_step(float* h, float* conv_state, const void* x_t, int x_dtype, const void* z_t, int z_dtype,
                    const float* delta_t, const float* B_t, const float* C_t, const float* A, const float* Dskip,
                    const float* conv_w, const float* conv_b, void* y_t, int y_dtype, int64_t batch, int64_t dim,
                    int dstate, int dconv, uint32_t flags, samba_stream_t stream) {
  const char* who = "samba_scan_step";
  if (!h || !x_t || !delta_t || !B_t || !C_t || !A || !y_t)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: h, x_t, delta_t, B_t, C_t, A and y_t are required", who);
  if (batch < 1 || dim < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (batch > 65535) return fail(SAMBA_ERR_UNSUPPORTED, "%s: batch above 65535", who);
  if (dstate != 4 && dstate != 8 && dstate != 16) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dstate", who);
  if (dconv < 2 || dconv > 4) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dconv must be 2..4", who);
  if (!dtype_ok(x_dtype) || !dtype_ok(y_dtype) || (z_t && !dtype_ok(z_dtype)))
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: dtype", who);
  if ((flags & SAMBA_SCAN_FUSE_CONV) && (!conv_state || !conv_w))
    return fail(SAMBA_ERR_INVALID_ARG, "%s: FUSE_CONV needs conv_state and conv_w", who);
  if (flags & ~7u) return fail(SAMBA_ERR_INVALID_ARG, "%s: unknown flag bits", who);
  return launch_scan_step(h, conv_state, x_t, x_dtype, z_t, z_dtype, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b,
                          y_t, y_dtype, batch, dim, dstate, dconv, flags, reinterpret_cast<cudaStream_t>(stream));
}

int samba_scan_carry(const float* h_in, const float* dsum, const float* A, const float* h_local, float* h_out,
                     int64_t batch, int64_t dim, int dstate, samba_stream_t stream) {
  const char* who = "samba_scan_carry";
  if (!dsum || !A || !h_local || !h_out) return fail(SAMBA_ERR_INVALID_ARG, "%s: dsum, A, h_local and h_out are required", who);
  if (batch < 1 || dim < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (dstate != 4 && dstate != 8 && dstate != 16) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dstate must be 4, 8 or 16", who);
  return launch_scan_carry(h_in, dsum, A, h_local, h_out, batch, dim, dstate, reinterpret_cast<cudaStream_t>(stream));
}

int samba_conv_state(const void* x, int x_dtype, const float* conv_state_in, float* conv_state_out, int64_t batch,
                     int64_t seqlen, int64_t dim, int dconv, samba_stream_t stream) {
  const char* who = "samba_conv_state";
  if (!x || !conv_state_out) return fail(SAMBA_ERR_INVALID_ARG, "%s: x and conv_state_out are required", who);
  if (batch < 1 || seqlen < 0 || dim < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (dconv < 2 || dconv > 4) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dconv must be 2..4", who);
  if (!dtype_ok(x_dtype)) return fail(SAMBA_ERR_UNSUPPORTED, "%s: dtype", who);
  if (conv_state_in && conv_state_in == conv_state_out)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: conv_state_out may not alias conv_state_in", who);
  return launch_conv_state(x, x_dtype, conv_state_in, conv_state_out, batch, seqlen, dim, dconv,
                           reinterpret_cast<cudaStream_t>(stream));
}

static int check_ring(int64_t batch, int heads_kv, int head_dim, int64_t window, const char* who) {
  if (batch < 1 || heads_kv < 1 || window < 1) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad shape", who);
  if (head_dim != 16 && head_dim != 32 && head_dim != 64 && head_dim != 128)
    return fail(SAMBA_ERR_UNSUPPORTED, "%s: head_dim must be 16, 32, 64 or 128", who);
  // The decode kernels index ring slots with 32-bit ints and put the KV heads
  // on a grid dimension of at most 65535 blocks.
  if (window > (int64_t(1) << 30)) return fail(SAMBA_ERR_UNSUPPORTED, "%s: window above 2^30", who);
  if (heads_kv > 65535) return fail(SAMBA_ERR_UNSUPPORTED, "%s: heads_kv above 65535", who);
  return SAMBA_OK;
}

// Shared checks of samba_swa_step and samba_swa_step_noalloc, in the order
// both report them.
static int check_swa_step(const void* q_t, const void* k_t, const void* v_t, const void* k_ring, const void* v_ring,
                          const int64_t* pos, const void* o_t, int64_t batch, int heads_q, int heads_kv,
                          int head_dim, int64_t window, const char* who) {
  if (!q_t || !k_t || !v_t || !k_ring || !v_ring || !pos || !o_t)
    return fail(SAMBA_ERR_INVALID_ARG, "%s: null pointer", who);
  int rc = check_ring(batch, heads_kv, head_dim, window, who);
  if (rc != SAMBA_OK) return rc;
  if (heads_q < 1 || heads_q % heads_kv != 0) return fail(SAMBA_ERR_INVALID_ARG, "%s: heads_q %% heads_kv", who);
  if (heads_q / heads_kv > 16) return fail(SAMBA_ERR_UNSUPPORTED, "%s: heads_q / heads_kv must be <= 16", who);
  if (batch > 65535) return fail(SAMBA_ERR_UNSUPPORTED, "%s: batch above 65535", who);
  const void* ptrs[] = {q_t, k_t, v_t, k_ring, v_ring, o_t};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  return SAMBA_OK;
}

int samba_swa_ring_fill(const void* k, const void* v, int64_t seqlen, void* k_ring, void* v_ring, int64_t* pos,
                        int64_t batch, int heads_kv, int head_dim, int64_t window, samba_stream_t stream) {
  const char* who = "samba_swa_ring_fill";
  if (!k || !v || !k_ring || !v_ring || !pos) return fail(SAMBA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (seqlen < 0) return fail(SAMBA_ERR_INVALID_ARG, "%s: bad seqlen", who);
  int rc = check_ring(batch, heads_kv, head_dim, window, who);
  if (rc != SAMBA_OK) return rc;
  const void* ptrs[] = {k, v, k_ring, v_ring};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  return launch_ring_fill(k, v, seqlen, k_ring, v_ring, pos, batch, heads_kv, head_dim, window,
                          reinterpret_cast<cudaStream_t>(stream));
}

size_t samba_swa_step_workspace_size(int64_t batch, int heads_q, int head_dim, int64_t window) {
  if (batch < 1 || heads_q < 1 || head_dim < 1 || window < 1) return 0;
  return swa_step_workspace(batch, heads_q, head_dim, window);
}

int samba_swa_step(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                   void* o_t, int64_t batch, int heads_q, int heads_kv, int head_dim, int64_t window, float scale,
                   void* workspace, size_t workspace_bytes, samba_stream_t stream) {
  const char* who = "samba_swa_step";
  int rc = check_swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, batch, heads_q, heads_kv, head_dim, window, who);
  if (rc != SAMBA_OK) return rc;
  const size_t need = swa_step_workspace(batch, heads_q, head_dim, window);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(SAMBA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", who, need, workspace_bytes);
  if (workspace && !aligned16(workspace)) return fail(SAMBA_ERR_INVALID_ARG, "%s: misaligned workspace", who);
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  return launch_swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, batch, heads_q, heads_kv, head_dim, window,
                         scale, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int samba_swa_step_noalloc(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring,
                           int64_t* pos, void* o_t, int64_t batch, int heads_q, int heads_kv, int head_dim,
                           int64_t window, float scale, samba_stream_t stream) {
  const char* who = "samba_swa_step_noalloc";
  int rc = check_swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, batch, heads_q, heads_kv, head_dim, window, who);
  if (rc != SAMBA_OK) return rc;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  return launch_swa_step_noalloc(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, batch, heads_q, heads_kv, head_dim, window,
                                 scale, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
