/*
 * vi.h -- C ABI of libvi, the B200 (sm_100a) kernels for the clip-parallel
 * temporal modules of a video-diffusion U-Net (Video-Infinity).
 *
 * Source of every operation: "Video-Infinity: Distributed Long Video
 * Generation" (write-up on news.43zhubao.com), the paragraphs on clip
 * parallelism and on the three temporal modules: dual-domain attention, the
 * temporal convolution, and GroupNorm.  The pages distribute the N clips of a
 * video over N GPUs and synchronise context between them; here all N clips
 * live on one GPU and each call partitions them inside one kernel grid (the
 * *_shard calls at the end serve a video spread over several GPUs).
 *
 * Common conventions
 * ------------------
 * Layout.  Every activation (q, k, v, out, x, y) is a dense row-major array
 *   [P positions][F frames][C channels], C innermost, with C = heads * d for
 *   attention.  P = H'*W' is the latent's spatial size.  Frames of one
 *   position are contiguous, so a clip and its neighbours are adjacent.
 * Clips.  F frames are cut into N clips of L = F / N frames; F % N == 0.
 * Types.  The un-suffixed entry points take bf16 tensors (IEEE bfloat16, bit
 *   patterns in uint16 storage) and accumulate in fp32; the _f32 entry points
 *   take fp32 tensors and compute in fp32 on CUDA cores (no TF32).  Small
 *   parameter vectors (conv weight and bias, GroupNorm gamma and beta) have
 *   the same type as the activations.
 * Pointers.  Every array pointer is a DEVICE pointer on the current CUDA
 *   device, 16-byte aligned, owned by the caller before and after the call.
 *   The library keeps no pointer after the call returns.
 * Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Calls enqueue work on it and return without synchronising; the outputs
 *   are ready when the stream reaches that point.  Scratch memory the library
 *   needs is taken, in stream order on that stream, from a memory pool the
 *   library creates for each device on first use (cudaMallocFromPoolAsync /
 *   cudaFreeAsync); the pool keeps up to 64 MiB of freed memory mapped so
 *   later calls reuse it.  Calls on different streams may run concurrently;
 *   calls on one stream run in order.
 * Empty calls.  P == 0 (no positions) is a valid call with nothing to
 *   compute: once the scalar arguments pass their checks it returns VI_OK,
 *   enqueues nothing and reads no pointer (they may be NULL).  F, N, C and the
 *   other sizes must still be positive.
 * Errors.  Every argument is checked on the host before anything is launched;
 *   a failed check returns a negative vi_status and enqueues nothing.
 *   VI_ERR_CUDA reports a CUDA error seen while launching.  A fault that
 *   happens on the device later surfaces, as usual in CUDA, at the caller's
 *   next synchronisation.
 */
#ifndef VI_H_
#define VI_H_

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                 /* == cudaStream_t's pointee */
typedef struct CUstream_st* vi_stream_t;

typedef enum {
  VI_OK = 0,
  VI_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, F % N != 0, ... */
  VI_ERR_ALIGNMENT = -2,    /* pointer not 16-byte aligned, or C * sizeof(T) % 16 != 0 */
  VI_ERR_UNSUPPORTED = -3,  /* valid request outside what the library implements */
  VI_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed while enqueuing */
  VI_ERR_DEVICE_TIMEOUT = -5  /* a kernel's bounded wait ran out (see vi_take_device_errors) */
} vi_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* vi_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int vi_version(void);

/*
 * Kernels that wait on an asynchronous copy or tensor-core operation bound
 * that wait (2 s of device time); when it runs out they record the fact in a
 * device-side error word and return early instead of hanging the GPU.  This
 * call synchronises the current device, reads and clears that word, and
 * returns VI_OK if no wait ran out since the last call, VI_ERR_DEVICE_TIMEOUT
 * otherwise (or VI_ERR_CUDA if the synchronisation itself failed).
 */
int vi_take_device_errors(void);

/*
 * Number of CUDA kernels this library has launched in the calling process
 * since it was loaded (all devices and streams; a diagnostic for profiling
 * and benchmarks, not an ordering primitive).
 */
unsigned long long vi_launch_count(void);

/*
 * Self-test of the bounded-wait path: enqueues one tiny kernel that waits on
 * an mbarrier nothing ever arrives at, gives up after limit_us microseconds
 * (1 .. 1000000), records the timeout in the device error word and returns.
 * The next vi_take_device_errors() then reports VI_ERR_DEVICE_TIMEOUT.  No
 * fault, trap or hang is involved; the GPU context stays usable.
 */
int vi_selftest_wait_timeout(int limit_us, vi_stream_t stream);

/*
 * Dual-domain temporal attention (attention-module paragraph of the source).
 *
 * For every position p, head h and clip i (frames [s, e), s = i*L, e = s+L),
 * each query frame f in [s, e) attends over the clip's key/value frame list
 *   own clip      s .. e-1
 *   C_pre         s-n_pre .. s-1          only if i > 0     (end of clip i-1)
 *   C_post        e .. e+n_post-1         only if i < N-1   (start of clip i+1)
 *   C_global      j * floor(F/n_global)   for j < n_global  (same for all clips)
 * concatenated without de-duplication (a frame listed twice counts twice):
 *   out[p,f,h,:] = sum_j softmax_j(q[p,f,h,:].k[p,j,h,:] / sqrt(d)) v[p,j,h,:]
 * Absent context at the video ends is left out of the softmax (not zero keys).
 *
 * q, k, v, out : [P][F][heads*d] (bf16, or fp32 for _f32); out must not
 *                overlap q, k or v.
 * Requirements : all sizes > 0 except P (>= 0) and the context sizes (>= 0); F % N == 0;
 *                d == 64; if N > 1 then n_pre <= L and n_post <= L;
 *                n_global <= F.  Otherwise VI_ERR_INVALID_ARG, or
 *                VI_ERR_UNSUPPORTED for d != 64.
 * Paths        : bf16 with n_global <= 16 and either L == 16 with n_pre,
 *                n_post <= 16 or L == 8 or 32 with n_pre, n_post <= 8 runs
 *                on tensor cores (TMA-staged blocks, mma.sync; an 8-row
 *                window on each side when both context sizes are <= 8, else
 *                16 rows; clips of 8 frames two to a warp, of 32 two warps
 *                to a clip); every other shape, and _f32, on CUDA cores, one
 *                warp per query frame (correct, much slower).
 * Scratch      : none.
 */
int vi_dual_attn(const void* q, const void* k, const void* v, void* out, int F, int N, int P,
                 int heads, int d, int n_pre, int n_post, int n_global, vi_stream_t stream);
int vi_dual_attn_f32(const void* q, const void* k, const void* v, void* out, int F, int N, int P,
                     int heads, int d, int n_pre, int n_post, int n_global, vi_stream_t stream);

/*
 * Temporal convolution with neighbour padding (conv-module paragraph).
 *
 * Each clip is extended by n = k/2 frames on each side, taken from the end of
 * the previous clip and the start of the next one, with zeros at the two ends
 * of the video; a valid cross-correlation over the extended clip gives
 *   y[p,f,co] = b[co] + sum_{t<k} sum_ci w[co,ci,t] * x[p, f+t-n, ci]
 * with x = 0 outside [0, F).  Because the neighbours' frames are exactly the
 * frames the unpartitioned sequence has there, the result equals the
 * zero-padded Conv1d of the whole video, and does not depend on N.
 *
 * x, y : [P][F][C];  w : [C_out=C][C_in=C][k] (PyTorch Conv1d order);  b : [C].
 * Requirements : sizes > 0 (P >= 0); F % N == 0; k odd; k/2 <= L; y must not overlap
 *                x, w or b.  Otherwise VI_ERR_INVALID_ARG.
 * Scratch      : the bf16 path repacks w into a stream-ordered scratch buffer
 *                of k*C*C*2 bytes (library pool), freed on the stream after
 *                the kernel.
 */
int vi_temporal_conv(const void* x, const void* w, const void* b, void* y, int F, int N, int P,
                     int C, int k, vi_stream_t stream);
int vi_temporal_conv_f32(const void* x, const void* w, const void* b, void* y, int F, int N,
                         int P, int C, int k, vi_stream_t stream);

/*
 * GroupNorm with global statistics (GroupNorm-module paragraph).
 *
 * Group g holds the C/groups contiguous channels [g*C/G, (g+1)*C/G).  Its mean
 * mu_g is aggregated over every clip (all frames, all positions); the spread
 * about that global mean is then aggregated over every clip into the global
 * variance var_g (biased: divided by the element count).  Each element is
 *   y = (x - mu_g) / sqrt(var_g + eps) * gamma[c] + beta[c]
 * which equals GroupNorm (batch 1) of the unpartitioned latent for any N.
 *
 * x, y : [P][F][C] (y may equal x: in place);  gamma, beta : [C].
 * Requirements : sizes > 0 (P >= 0); F % N == 0; C % groups == 0; eps >= 0 and finite.
 *                y may alias x exactly but must not partly overlap it.
 * Scratch      : (24 * groups * blocks + 16*C + 16*groups + 64) bytes of stream-ordered
 *                scratch (library pool) for per-block partial sums and the
 *                per-channel coefficients, freed on the stream after the last
 *                kernel.
 */
int vi_groupnorm_global(const void* x, const void* gamma, const void* beta, void* y, int F, int N,
                        int P, int C, int groups, float eps, vi_stream_t stream);
int vi_groupnorm_global_f32(const void* x, const void* gamma, const void* beta, void* y, int F,
                            int N, int P, int C, int groups, float eps, vi_stream_t stream);

/*
 * Temporal attention module: input projections, dual-domain attention, output
 * projection (bf16).  The attention-module paragraph redefines how the keys and
 * values are gathered (the module changes its K/V computation); the projections
 * around it are the module's linear layers:
 *   q = x Wq^T + bq,  k = x Wk^T + bk,  v = x Wv^T + bv      (per frame)
 *   a = vi_dual_attn(q, k, v; heads, d, n_pre, n_post, n_global)
 *   out = a Wo^T + bo
 * The three input projections are ONE tensor-core GEMM of N = 3C over x
 * (the temporal-conv kernel with a single tap, its output channels split
 * into the q, k and v tensors), each written as a bf16 tensor.  Then, where
 * C <= 320 and the attention takes its tensor-core path with n_pre, n_post
 * <= 8, one kernel runs the attention and the output projection (a is
 * rounded to bf16 on chip and never written); otherwise the attention kernel
 * writes a (bf16) and the output projection GEMM follows.  The two forms
 * differ only in the fp32 summation order of the output projection.
 *
 * x, out : [P][F][C], C = heads*d;  w_qkv : [3C][C] (rows Wq, Wk, Wv, PyTorch
 * Linear layout);  b_qkv : [3C];  w_out : [C][C];  b_out : [C].
 * workspace : device buffer of vi_temporal_attention_workspace_bytes(F, P, C)
 *             bytes (16-byte aligned), owned by the caller, holding q, k, v
 *             (and a, when the projection is not fused) between the stages;
 *             contents undefined after the call.
 * Requirements : those of vi_dual_attn; C % 64 == 0; out, x, weights and
 *                workspace must not overlap.
 */
unsigned long long vi_temporal_attention_workspace_bytes(int F, int P, int C);
int vi_temporal_attention(const void* x, const void* w_qkv, const void* b_qkv, const void* w_out,
                          const void* b_out, void* out, void* workspace, int F, int N, int P,
                          int heads, int d, int n_pre, int n_post, int n_global,
                          vi_stream_t stream);

/*
 * GroupNorm with global statistics followed by the temporal convolution,
 * fused (bf16).  The ResNet module of the write-up normalises and then
 * convolves along frames (GroupNorm-module and conv-module paragraphs);
 *   y = conv(GroupNorm(x; gamma, beta, groups, eps); w, b)
 * computed without writing the normalised tensor to memory: one statistics
 * pass over x gives per-channel (m_c, a_c = gamma_c / sigma_g, beta_c); the
 * tensor-core conv then runs on the raw x with the weights scaled per input
 * channel, W'[co][ci][t] = bf16(w[co][ci][t] a_ci), and per-output-channel
 * bias tables b[co] + sum over the taps inside the video of
 * sum_ci (w beta_ci - W' m_ci), computed in fp64 from the same rounded W' (so
 * the mean terms cancel exactly).  The zero padding at the video ends applies
 * to the NORMALISED sequence: frames within k/2 of an end take the table of
 * their valid taps.  The result differs from the two bf16 calls composed by
 * bf16 rounding (of W a instead of the normalised tensor).
 *
 * x, y : [P][F][C];  gamma, beta, b : [C];  w : [C][C][k].
 * Requirements : those of vi_groupnorm_global and vi_temporal_conv; y must
 *                not overlap any input; the fused kernel also needs
 *                C % 64 == 0 and k <= 7 (VI_ERR_UNSUPPORTED otherwise).
 * Scratch      : GroupNorm statistics, folded w and the bias tables (library
 *                pool).
 */
int vi_groupnorm_conv(const void* x, const void* gamma, const void* beta, const void* w,
                      const void* b, void* y, int F, int N, int P, int C, int groups, float eps,
                      int k, vi_stream_t stream);

/*
 * GroupNorm with global statistics that allocates nothing (bf16 only).
 *
 * The source paper has no counterpart to this entry point.  It is for callers
 * that cannot allocate device memory while they run -- for example a plugin
 * inside an inference engine that owns all device memory and forbids
 * allocation in its execution step, or a service whose memory footprint is
 * fixed when it starts -- and therefore cannot use vi_groupnorm_global, which
 * takes its scratch from a stream-ordered allocator.  The caller still provides every
 * input and output.
 *
 * Arguments, layout, result and argument checks: as vi_groupnorm_global.
 * Scratch      : a 1 MiB array inside libvi (a static __device__ array that
 *                every GPU which loads the library holds until the process
 *                exits).  A call whose scratch need is larger returns
 *                VI_ERR_UNSUPPORTED before launching anything.  The need is
 *                64 + 16*groups + 16*C + 24*groups*B bytes (each term rounded
 *                up to 64 bytes), B being the partial-sum records per group:
 *                at most the SM count on the streaming path, and at most
 *                8*SMs/groups + 1 on the path for rows of more than 960
 *                16-byte vectors or 32 KB, or groups that split a 16-byte
 *                vector (there the last term is at most 24*(8*SMs + groups)).
 *                On a 148-SM B200 the streaming path admits, e.g., 32 groups
 *                with C up to ~58000 or 256 groups with C up to ~8000.
 * First call   : the first call on each device looks up the array's device
 *                address with that device current (cudaGetSymbolAddress) and
 *                caches it.  It may also load the library's GPU code (CUDA
 *                loads modules lazily), which allocates device memory.  A
 *                caller whose running phase must not allocate should therefore
 *                make one call during its setup, before any stream capture;
 *                later calls allocate nothing.
 * Sharing      : every call uses the same array.  Each call clears the part
 *                that must start at zero and rewrites the rest, but calls
 *                whose work overlaps on the GPU (different streams, or several
 *                host threads) race on it and give wrong results: serialise
 *                them, e.g. on one stream.
 */
int vi_groupnorm_global_noalloc(const void* x, const void* gamma, const void* beta, void* y,
                                int F, int N, int P, int C, int groups, float eps,
                                vi_stream_t stream);

/*
 * ---- Shards of a video cut along frames (clip parallelism over GPUs) ----
 *
 * Source: the write-up's clip-parallelism paragraphs: each device holds some
 * clips of the video and receives, before its temporal modules run, the
 * frames its clips need from the neighbouring devices (the end of the previous
 * clip and the start of the next) and the globally sampled frames, and the
 * devices exchange GroupNorm statistics.  These calls are the per-device
 * compute of that scheme; the exchange itself is the caller's (NCCL, or the
 * package's ClipParallel).  A shard holds F_loc consecutive frames of every
 * position; bf16 only.
 *
 * Halo-padded storage: the tensors whose neighbour frames a module reads
 * (k and v of the attention, x of the conv) are taken as [P][F_loc + 2h][C]
 * with the shard's frames at rows [h, h + F_loc) and h spare rows on each
 * side.  The caller keeps its shard in that layout, and the exchange writes
 * only the 2h halo rows of each position (zeros at the video ends), so no
 * call copies the shard.
 *
 * part: which frame blocks a call computes.  VI_PART_ALL computes the whole
 * shard.  VI_PART_INTERIOR computes only the blocks whose reads stay inside
 * the shard's own frames (no halo row is read, so the call may run while the
 * halo exchange is still in flight); VI_PART_BOUNDARY computes the others.
 * INTERIOR followed by BOUNDARY gives the result of ALL.  A part with no
 * block (e.g. INTERIOR of a shard of one block) is a valid empty call.
 */
enum { VI_PART_ALL = 0, VI_PART_INTERIOR = 1, VI_PART_BOUNDARY = 2 };

/*
 * Dual-domain attention of one shard (attention-module paragraph).
 *
 * q, out        : [P][F_loc][C], the shard's frames: clips clip0 ..
 *                 clip0 + N_loc - 1 of the video's N clips (L = F_loc / N_loc).
 * k_ext, v_ext  : [P][F_loc + 16][C], halo-padded (h = 8): the 8 frames before
 *                 the shard, the shard's F_loc frames, the 8 frames after it.
 *                 Rows past a video end are masked out but are read: they must
 *                 hold finite values (zeros).
 * k_glob, v_glob: [P][n_global][C]: the video's global frames
 *                 j * floor(F / n_global), j < n_global (unused if n_global == 0).
 * part         : VI_PART_*; a block is 8 clips (128 frames), the boundary
 *                 blocks are the first and the last.
 * Result       : exactly vi_dual_attn of the whole video, restricted to the
 *                 shard's frames (the part's blocks of them).
 * Requirements : L == 16, d == 64, n_pre, n_post <= 8, n_global <= 16
 *                 (VI_ERR_UNSUPPORTED otherwise); 0 <= clip0 <= N - N_loc;
 *                 part in 0..2; out must not overlap any input; P == 0 is an
 *                 empty call.
 */
int vi_dual_attn_shard(const void* q, const void* k_ext, const void* v_ext, const void* k_glob,
                       const void* v_glob, void* out, int F_loc, int N_loc, int clip0, int N,
                       int P, int heads, int d, int n_pre, int n_post, int n_global, int part,
                       vi_stream_t stream);

/*
 * Temporal conv of one shard (conv-module paragraph: each clip padded with
 * the neighbours' boundary frames).
 *
 * x_ext : [P][F_loc + 2*(k/2)][C], halo-padded (h = k/2): k/2 frames before
 *         the shard (zeros at the start of the video), the shard's frames,
 *         k/2 frames after it (zeros at the end).   y : [P][F_loc][C].
 *         w : [C][C][k];  b : [C].
 * part  : VI_PART_*; a block is 128 frames; the interior blocks are those
 *         whose frames and k/2 neighbours on each side lie in the shard.
 * Result       : vi_temporal_conv of the whole video on the shard's frames
 *                (the part's blocks of them).
 * Requirements : k odd; the tensor-core path (C % 64 == 0), else
 *                VI_ERR_UNSUPPORTED; part in 0..2; y must not overlap x_ext,
 *                w or b.
 */
int vi_temporal_conv_shard(const void* x_ext, const void* w, const void* b, void* y, int F_loc,
                           int P, int C, int k, int part, vi_stream_t stream);

/*
 * GroupNorm across shards (GroupNorm-module paragraph): every shard reduces
 * its rows (vi_groupnorm_shard_stats), the W shards' statistics are gathered
 * onto every device, and each shard normalises its rows with the merged
 * statistics (vi_groupnorm_shard_apply).  All shards must hold the same
 * number of rows (F_loc * P).
 *
 * stats       : [groups][2] fp64 device array, (mean, var) of this shard's rows
 *               (biased variance).
 * shard_stats : [W][groups][2], the W shards' stats in any order.  Merged as
 *               mean = average of the means, var = average of (var_w +
 *               (mean_w - mean)^2), which is the variance of the union.
 * Requirements : P > 0 (a shard with no rows has no statistics); C % groups
 *                == 0; groups <= 1024; y may equal x.
 */
int vi_groupnorm_shard_stats(const void* x, int F_loc, int P, int C, int groups, double* stats,
                             vi_stream_t stream);
int vi_groupnorm_shard_apply(const void* x, const double* shard_stats, int W, const void* gamma,
                             const void* beta, void* y, int F_loc, int P, int C, int groups,
                             float eps, vi_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VI_H_ */
