/*
 * zr.h -- C ABI of the fused ZeRO sharded optimizer step for NVIDIA B200
 * (sm_100a): stages 1 and 2, and the parameter side of stage 3.
 *
 * One step of data-parallel training with sharded optimizer state, for the
 * slice of parameters that one rank owns:
 *
 *   1. reduce   g = (g_0 + g_1 + ... + g_{W-1}) / W   -- the W replicas'
 *               bf16 gradients for the owned elements, summed in fp32 in
 *               rank order, then divided by W.  This is the reduce half of
 *               the gradient reduce-scatter ("CS336 lecture 8, parallelism
 *               basics", ZeRO level 1 and its code sketch; "Scaling training
 *               to thousands of GPUs", 03:41 DP: gradients are summed and
 *               averaged over replicas; 11:24 ZeRO: AllReduce is
 *               reduce-scatter + all-gather);
 *   2. clip     optional: g <- g * min(1, max_norm / (||g||_global + 1e-6))
 *               (not on those pages; the usual global-norm convention);
 *   3. AdamW    on the owned slice's fp32 master weights p and moments m, v
 *               (the pages name AdamW with fp32 master / m / v -- "DDP -> ZeRO"
 *               blog section 1.1, "CS336" 16 bytes/param ledger; the rule is
 *               bias-corrected Adam with decoupled weight decay):
 *                 m = b1*m + (1-b1)*g ;  v = b2*v + (1-b2)*(g*g)
 *                 p = p*(1 - lr*wd)
 *                 p = p - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps)
 *   4. cast     param_out[global position] = bf16(p), round to nearest even:
 *               this rank's contribution to the parameter all-gather buffer
 *               ("CS336", ZeRO-1 sketch, update-then-gather).
 *
 * The four stages run as one fused, memory-bound GPU pass (two passes and a
 * small combine kernel when clipping).  The W replicas' gradients live in
 * memory the GPU can load from: its own, or other GPUs' buffers mapped with
 * CUDA IPC (zr_ipc_*).  There is no collective: the reduce-scatter and the
 * all-gather are the kernel's own loads and stores.
 *
 * Partitioning ("Scaling training to thousands of GPUs", 11:24 ZeRO, FSDP1
 * vs FSDP2):
 *   ZR_PARTITION_FLAT          tensors concatenated in declaration order and
 *                              zero padded to W equal chunks of
 *                              C = ceil(N/W); rank r owns [r*C, (r+1)*C).
 *   ZR_PARTITION_WHOLE_TENSOR  every tensor owned whole by one rank, greedy
 *                              longest-processing-time balance by element
 *                              count (largest first, ties by declaration
 *                              index; to the least-loaded rank, ties by
 *                              lowest rank).  No padding.
 * Buckets ("Scaling training ...", 03:41 DP, bucket_cap_mb; "DDP -> ZeRO"
 * blog section 2.1): whole tensors packed in reverse declaration order; a new
 * bucket opens when the next tensor's bf16 gradient bytes would push a
 * non-empty bucket past bucket_cap_bytes.  The flat zero pad closes bucket 0.
 *
 * Layouts
 *   global layout  all tensors, declaration order, flat (plus the flat pad);
 *                  param_out is a bf16 buffer of padded_numel elements in it.
 *   owned order    the order of this rank's elements: flat -> [r*C, (r+1)*C)
 *                  as is; whole-tensor -> this rank's tensors in declaration
 *                  order, concatenated.  master, m, v and every grad_ptrs[w]
 *                  hold owned_numel elements in owned order.
 *
 * Ownership and errors
 *   The caller allocates and owns every device buffer, including the
 *   workspace; a plan owns host memory only.  Device-side calls are
 *   asynchronous on the given stream and return the launch status; a fault
 *   inside a kernel surfaces at the caller's next synchronisation.  On any
 *   error status nothing has been launched.  Buffers must not overlap; the
 *   gradient buffers are read-only.  A plan may be used from one host thread
 *   at a time, and only while the device that was current when its
 *   workspace was bound is current (else ZR_ERR_INVALID_ARG).
 */
#ifndef ZR_H_
#define ZR_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* zr_stream_t;

typedef enum {
    ZR_OK = 0,
    ZR_ERR_INVALID_ARG = 1,   /* bad size, rank, mode, step, NULL pointer    */
    ZR_ERR_ALIGNMENT = 2,     /* a device pointer not 16-byte aligned        */
    ZR_ERR_NO_WORKSPACE = 3,  /* zr_plan_set_workspace not called / too small */
    ZR_ERR_CUDA = 4,          /* a CUDA runtime call failed                  */
    ZR_ERR_UNSUPPORTED = 5,   /* W above ZR_MAX_WORLD_SIZE, no sm_100 device */
    ZR_ERR_BUFFER_TOO_SMALL = 6,
    ZR_ERR_IO = 7,            /* a checkpoint file could not be read or written */
    ZR_ERR_MISMATCH = 8       /* a checkpoint does not belong to this plan, or is corrupt */
} zr_status;

typedef enum { ZR_PARTITION_FLAT = 0, ZR_PARTITION_WHOLE_TENSOR = 1 } zr_partition;

/* Largest W: the W gradient pointers travel by value in the kernel's
 * parameter block. */
#define ZR_MAX_WORLD_SIZE 512

/* AdamW hyperparameters (fp32, as a training script holds them).
 * max_grad_norm <= 0 disables clipping. */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay, max_grad_norm;
} zr_adamw;

/* One piece of the partition: a run of `length` consecutive elements of
 * tensor `tensor` (-1: the flat zero pad), starting at element
 * `offset_in_tensor`, placed in bucket `bucket`, owned by rank `owner`, at
 * `global_offset` in the global layout and `owned_offset` in the owner's
 * owned order.  Segments are ordered by bucket, then by tensor in packing
 * (reverse declaration) order, then by offset; the pad comes last in
 * bucket 0. */
typedef struct {
    int32_t bucket, tensor, owner, reserved;
    int64_t offset_in_tensor, length, global_offset, owned_offset;
} zr_segment;

typedef struct zr_plan zr_plan;

/* Build the partition, bucket and segment tables for one rank (host only,
 * no CUDA call).  n_tensors >= 0; ndims[t] >= 0; shapes[t] points to
 * ndims[t] non-negative extents (a tensor of ndims 0 is a scalar).
 * 1 <= world_size <= ZR_MAX_WORLD_SIZE, 0 <= rank < world_size.
 * bucket_cap_bytes counts bf16 gradient bytes (2 per element).  *hp is
 * copied.  On success *out receives a plan to release with zr_plan_destroy.
 * Errors: ZR_ERR_INVALID_ARG (NULL pointers, negative extents, bad mode or
 * rank, element counts overflowing int64), ZR_ERR_UNSUPPORTED (W too large). */
zr_status zr_plan_create(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                         int32_t world_size, int32_t rank, zr_partition mode,
                         uint64_t bucket_cap_bytes, const zr_adamw* hp, zr_plan** out);

/* zr_plan_create with buckets given by tensor groups instead of a byte cap:
 * tensor_group[t] (n_tensors entries, non-decreasing in declaration order)
 * names the unit tensor t belongs to -- typically its layer -- and every
 * group becomes one bucket, numbered in backward order (the last group is
 * bucket 0; the flat zero pad closes bucket 0 as usual).  The unit is the
 * ZeRO-3 / FSDP one ("CS336 lecture 8", FSDP sketch; "Scaling training to
 * thousands of GPUs", 11:24 ZeRO, stage 3): zr_step_bucket on a layer's
 * bucket reduces that layer's gradients, and updates its slice, as soon as
 * its backward has produced them.  Partition, owners, offsets and tiles are
 * those of zr_plan_create; only bucket ids and segment order differ.
 * Errors: as zr_plan_create, plus ZR_ERR_INVALID_ARG (tensor_group NULL
 * with n_tensors > 0, or decreasing). */
zr_status zr_plan_create_grouped(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                                 const int32_t* tensor_group, int32_t world_size, int32_t rank,
                                 zr_partition mode, const zr_adamw* hp, zr_plan** out);

/* Sizes of the plan.  Any output pointer may be NULL.  owned_numel is this
 * rank's element count; n_segments counts all ranks' segments. */
zr_status zr_plan_query(const zr_plan* plan, int64_t* total_numel, int64_t* padded_numel,
                        int64_t* owned_numel, int32_t* n_buckets, int64_t* n_segments);

/* Copy all ranks' segments (see zr_segment) into out[0..cap).  *n receives
 * the total count; if it exceeds cap, nothing is written and
 * ZR_ERR_BUFFER_TOO_SMALL is returned (call with cap 0 to size). */
zr_status zr_plan_segments(const zr_plan* plan, zr_segment* out, int64_t cap, int64_t* n);

/* Device workspace the plan needs: the tile tables, the clip partial sums
 * (one double per tile, one per group of 1024 tiles, and a completion
 * counter), a few scalars and status words, the ZeRO-3 gather
 * piece table (32 bytes per piece of at most 16384 elements, all ranks) and
 * (when clipping with W > 4, or with a grouped plan) an fp32 scratch copy
 * of the reduced gradient. */
zr_status zr_plan_workspace_bytes(const zr_plan* plan, uint64_t* bytes);

/* Bind a device workspace (>= zr_plan_workspace_bytes, 256-byte aligned,
 * owned by the caller, kept alive while the plan is used) and upload the
 * tile tables and the gather piece table into it with asynchronous copies
 * on `stream` (clearing checked mode's status and the clip's counter).  Selects the
 * current CUDA device as the plan's device.  Errors: ZR_ERR_NO_WORKSPACE
 * (too small), ZR_ERR_ALIGNMENT, ZR_ERR_UNSUPPORTED (the current device is
 * not compute capability 10.x), ZR_ERR_CUDA. */
zr_status zr_plan_set_workspace(zr_plan* plan, void* d_workspace, uint64_t bytes,
                                zr_stream_t stream);

/* New AdamW hyperparameters for the calls that follow (a learning-rate
 * schedule changes lr every step; the pages' lr of 3e-4 is one constant
 * point of it).  Host-side: every step call computes its scalars from the
 * plan's current values, except that zr_step_device_count passes them by
 * value to its scalars kernel, so a CUDA graph that captured it keeps the
 * values current at capture.  Turning clipping on or off (max_grad_norm
 * crossing 0) changes what the workspace holds: ZR_ERR_UNSUPPORTED, make a
 * new plan.  Errors: ZR_ERR_INVALID_ARG (NULL), ZR_ERR_UNSUPPORTED. */
zr_status zr_plan_set_adamw(zr_plan* plan, const zr_adamw* hp);

/* A learning rate in device memory for zr_step_device_count: its scalars
 * kernel reads *d_lr (one fp32, caller-owned, 4-byte aligned) at every
 * launch instead of the plan's lr, so a captured graph follows a schedule
 * that the caller's own device work updates between replays.  NULL (the
 * default) goes back to the plan's lr.  The other hyperparameters stay
 * those current at capture.  Errors: ZR_ERR_INVALID_ARG, ZR_ERR_ALIGNMENT. */
zr_status zr_plan_set_device_lr(zr_plan* plan, const float* d_lr);

/* Clipping only.  d_partials: device array of world_size doubles, entry w =
 * rank w's sum of squares S_w of its averaged owned gradient.  zr_step
 * writes this rank's entry itself; the other entries must hold the other
 * ranks' S_w (from zr_grad_sumsq, or from a scalar all-gather across GPUs)
 * before zr_step runs on the stream.  The clip norm is
 * sqrt(S_0 + S_1 + ... + S_{W-1}), summed in rank order in fp64, so every
 * rank derives the same coefficient.
 * This array takes the place of a single pre-summed "other ranks' S"
 * scalar (a zr_plan_set_peer_sumsq(plan, d_peer_sumsq) form): with one such
 * scalar each rank would add its own S_r at a different position of the
 * sum, fp64 addition is not associative, and the ranks could clip by
 * coefficients that differ in the last bit.  With all W entries in one
 * array every rank forms the identical sum. */
zr_status zr_plan_set_sumsq_partials(zr_plan* plan, double* d_partials);

/* The optimizer step for this rank (stages 1-4 above).
 * grad_ptrs: host array of world_size device pointers, replica w's bf16
 *            gradient for this rank's owned elements in owned order.
 * master, m, v: fp32 device arrays of owned_numel, updated in place.
 * param_out: bf16 device array of padded_numel (global layout); only this
 *            rank's positions are written.  (With the ZR_PARAMS_OWNED
 *            layout, zr_plan_set_param_layout below: this rank's shard,
 *            owned_numel elements in owned order.)
 * step: 1-based AdamW step count t (bias corrections use it).
 * Every device pointer must be 16-byte aligned.  With owned_numel == 0 it
 * returns ZR_OK and launches nothing.
 * Errors: ZR_ERR_INVALID_ARG, ZR_ERR_ALIGNMENT, ZR_ERR_NO_WORKSPACE (also:
 * clipping enabled and no partials array bound), ZR_ERR_CUDA. */
zr_status zr_step(const zr_plan* plan, const void* const* grad_ptrs, float* master, float* m,
                  float* v, void* param_out, int64_t step, zr_stream_t stream);

/* zr_step for CUDA-graph capture: the step count lives in device memory.
 * *d_step (int64, device, 8-byte aligned) holds the number of steps already
 * taken; the call first advances it on the device and computes the AdamW
 * scalars there (fp64 from the fp32 hyperparameters, rounded once to fp32,
 * as zr_step does on the host), then runs the step as zr_step(t = new
 * count).  Nothing in it depends on host values that change from step to
 * step, so a graph that captured it replays as the next step each time.
 * Results equal zr_step's (device and host fp64 pow may differ in the last
 * fp64 place; after the rounding to fp32 the scalars agree except in rare
 * ties).  Errors: as zr_step. */
zr_status zr_step_device_count(const zr_plan* plan, const void* const* grad_ptrs, float* master,
                               float* m, float* v, void* param_out, int64_t* d_step,
                               zr_stream_t stream);

/* One bucket of the step, for overlapping the optimizer with the backward
 * pass ("Scaling training to thousands of GPUs", 03:41 DP: a bucket's
 * collective starts as soon as backward has produced its gradients;
 * "CS336 lecture 8", ZeRO level 2: a gradient is released as soon as it has
 * been reduced).  Enqueue it on a stream that waits for the bucket's
 * gradients (e.g. cudaStreamWaitEvent).  Arguments as zr_step, plus
 * 0 <= bucket < n_buckets; only this rank's elements of that bucket are read
 * and written, and a bucket this rank owns nothing of is a no-op.
 *   Without clipping: the fused step on the bucket's elements.  Calling it
 *   once per bucket, in any order, gives exactly zr_step's result (the step
 *   is elementwise).
 *   With clipping: the coefficient needs every bucket's sum of squares, so
 *   this runs the reduce and the sums of squares for the bucket (writing the
 *   fp32 averaged gradient to the workspace when W > 4 or the plan is
 *   grouped; master, m, v and
 *   param_out are not touched and may be NULL); after every bucket,
 *   zr_step_finish updates all elements.  For W > 4 (or a grouped plan)
 *   the bucket's gradient
 *   buffers may be released as soon as this call's work is done.
 * Errors: as zr_step; ZR_ERR_INVALID_ARG for a bucket out of range. */
zr_status zr_step_bucket(const zr_plan* plan, int32_t bucket, const void* const* grad_ptrs,
                         float* master, float* m, float* v, void* param_out, int64_t step,
                         zr_stream_t stream);

/* Completes a bucket-by-bucket step of a plan with clipping: the norm from
 * all buckets' sums of squares (and the other ranks' entries of the
 * partials array, as for zr_step), then the scaled AdamW update and bf16
 * cast of every owned element.  For W > 4 (or a grouped plan) it reads the
 * averaged gradient that zr_step_bucket stored and grad_ptrs may be NULL;
 * otherwise it reads
 * the gradients again, so grad_ptrs must still hold every bucket's values.
 * For plans without clipping it does nothing and returns ZR_OK.  The result
 * equals zr_step's bit for bit. */
zr_status zr_step_finish(const zr_plan* plan, const void* const* grad_ptrs, float* master, float* m,
                         float* v, void* param_out, int64_t step, zr_stream_t stream);

/* Between a bucket-by-bucket pass and zr_step_finish, with clipping: this
 * rank's S_r from the sums of squares zr_step_bucket left in the workspace
 * (every bucket of the step called once), to the device double *d_out,
 * without reading any gradient -- the value zr_step_finish will use for
 * this rank, bit for bit.  Its purpose is the cross-rank exchange of a
 * layer-by-layer step whose gradients are released as each layer is
 * reduced (ZeRO-3): every rank calls it, the W values are all-gathered into
 * the partials array, then zr_step_finish.  Errors: ZR_ERR_INVALID_ARG (no
 * clipping, NULL), ZR_ERR_ALIGNMENT (d_out not 8-byte aligned),
 * ZR_ERR_NO_WORKSPACE, ZR_ERR_CUDA. */
zr_status zr_bucket_sumsq(const zr_plan* plan, double* d_out, zr_stream_t stream);

/* zr_step with host-resident gradients and a host copy of the result, for
 * callers whose gradients arrive in host memory.  Copies host_grad_ptrs[w]
 * (owned_numel bf16, owned order; pinned host memory for asynchronous
 * copies) into dev_grad_ptrs[w], runs the step, and copies this rank's
 * positions of param_out into host_param_out (a host buffer in the global
 * layout, padded_numel bf16; in owned order, owned_numel bf16, with the
 * ZR_PARAMS_OWNED layout).  The owned range is cut into up to 4 chunks
 * (1/2, 1/4, 1/8, 1/8 of it): while one chunk's gradients cross PCIe,
 * earlier chunks are stepped and their parameters copied back, on two
 * internal copy streams of the plan
 * (created by the plan's first zr_step_host call, released by
 * zr_plan_destroy) joined to `stream` by events.  Results equal zr_step's.
 * Asynchronous: `stream` reaches the end of the call only when every copy is
 * done; the host buffers must stay untouched until then. */
zr_status zr_step_host(const zr_plan* plan, const void* const* host_grad_ptrs,
                       void* const* dev_grad_ptrs, float* master, float* m, float* v,
                       void* param_out, void* host_param_out, int64_t step, zr_stream_t stream);

/* Clipping building block: writes this rank's S_r = sum over owned elements
 * of g*g (g the averaged gradient, each square exact in fp64, fp64
 * accumulation in a fixed order) to the device double *d_out.  zr_step's
 * own pass computes bit-identical values, so other ranks' entries of the
 * partials array may come from this call. */
zr_status zr_grad_sumsq(const zr_plan* plan, const void* const* grad_ptrs, double* d_out,
                        zr_stream_t stream);

/* Test hook: write the averaged fp32 gradient g (stage 1 only, before any
 * clipping) for the owned elements, in owned order, to g_out (owned_numel
 * floats, 16-byte aligned). */
zr_status zr_debug_reduce(const zr_plan* plan, const void* const* grad_ptrs, float* g_out,
                          zr_stream_t stream);

/* Verification hook for the averaging of stage 1 (g = s / W, rounded to
 * nearest even; for a power-of-two W the kernels multiply by 1/W instead of
 * dividing, which is exact scaling).  Runs the kernels' averaging on every
 * one of the 2^32 fp32 bit patterns s for each W in [w_first, w_last]
 * (1 <= w_first <= w_last <= ZR_MAX_WORLD_SIZE) and compares the bits with
 * IEEE division on the GPU; d_mismatches[W - w_first] (device,
 * w_last - w_first + 1 uint64 counters, 8-byte aligned, zeroed by the call)
 * receives the number of inputs whose results differ, NaN against NaN
 * counting as equal.  Asynchronous on `stream`: one grid per W (about 10 ms
 * each on a B200).  Errors: ZR_ERR_INVALID_ARG, ZR_ERR_ALIGNMENT,
 * ZR_ERR_UNSUPPORTED (not compute capability 10.x), ZR_ERR_CUDA.  Needs no
 * plan. */
zr_status zr_debug_average_check(int32_t w_first, int32_t w_last, uint64_t* d_mismatches,
                                 zr_stream_t stream);

/* ---------------------------------------------------------------------
 * ZeRO across GPUs over peer memory (NVLink / NVSwitch), one process per GPU
 * ("CS336 lecture 8", ZeRO-1 sketch: reduce-scatter of the gradients, update
 * of the owned slice, all-gather of the updated parameters).  The same
 * fused kernel does all three: grad_ptrs may point into other GPUs' memory
 * (peer loads are the reduce-scatter), and with gather targets set, every
 * bf16 result is stored into every rank's parameter buffer (peer stores are
 * the all-gather).  Ordering between ranks is the caller's: every replica's
 * gradients must be complete before any rank's step starts, and no rank may
 * read its parameter buffer before every rank's step has completed (for
 * example: synchronise the stream, then a process-group barrier, on both
 * sides).  Nothing in the kernels waits on another GPU.
 * ------------------------------------------------------------------- */

/* Owner-major layout of a full gradient buffer: rank r's owned elements, in
 * its owned order, start at offsets[r]; each rank's region is rounded up to
 * a multiple of 8 elements so that every region starts 16-byte aligned;
 * offsets[W] is the buffer's length in elements.  (In the flat mode with a
 * chunk that is a multiple of 8 this is exactly the global layout.)  When
 * every replica keeps its full gradient in this layout, the pointer to
 * replica w's buffer plus offsets[r] elements is what rank r passes as
 * grad_ptrs[w].  offsets: world_size + 1 entries. */
zr_status zr_plan_owner_offsets(const zr_plan* plan, int64_t* offsets);

/* Make zr_step, zr_step_device_count, zr_step_bucket and zr_step_finish
 * store each bf16 result in targets[0..world_size) (rank w's parameter
 * buffer, global layout, local or peer-mapped, 16-byte aligned) instead of
 * param_out, which may then be NULL.  The pointer array is copied into the
 * workspace (synchronising `stream`); targets == NULL goes back to
 * param_out.  zr_step_host refuses a plan with gather targets
 * (ZR_ERR_UNSUPPORTED); zr_step_no_alloc always writes param_out alone.
 * Needs a bound workspace. */
zr_status zr_plan_set_gather_targets(zr_plan* plan, void* const* targets, zr_stream_t stream);

/* A device buffer as another process can map it: the CUDA IPC handle of the
 * allocation that holds it and the buffer's offset in that allocation. */
typedef struct {
    unsigned char handle[64];
    uint64_t offset;
    uint64_t allocation_bytes;
} zr_ipc_handle;

/* zr_ipc_export: describe device_ptr (any address inside a cudaMalloc
 * allocation of this process) for another process.  zr_ipc_open: map a
 * handle exported by another process (same or other GPU; peer access is
 * enabled as needed) and return the buffer's address; release it with
 * zr_ipc_close.  A process cannot open its own handles (use the pointer).
 * Errors: ZR_ERR_INVALID_ARG, ZR_ERR_CUDA (no GPU driver, memory that IPC
 * cannot share such as virtual-memory-management allocations). */
zr_status zr_ipc_export(const void* device_ptr, zr_ipc_handle* out);
zr_status zr_ipc_open(const zr_ipc_handle* handle, void** device_ptr);
zr_status zr_ipc_close(void* device_ptr);

/* Checkpoints of the sharded optimizer state ("DDP -> ZeRO -> TP/PP/CP"
 * blog, section 3.3: sharded state must be gathered to be saved as a whole
 * model).  One file per rank: a 256-byte header -- magic "ZRSHARD1",
 * version 1, W, rank, mode, element counts, a hash of the tensors and one of
 * the partition (tensors, W, mode), the step, the AdamW hyperparameters and
 * a 64-bit FNV-1a checksum of the payload -- then master, m and v (fp32,
 * owned order).  The bf16 parameters need no checkpoint of their own: after
 * a step the all-gather buffer param_out already holds them whole.
 *
 * zr_state_save: copies this rank's master, m, v (device, owned_numel fp32
 * each) to the host after the work queued on `stream` (it synchronises the
 * stream) and writes them with `step` to `path` (through a temporary file
 * renamed into place).  zr_state_load: reads `path`, checks that it belongs
 * to this plan's partition and rank and that its checksum holds, copies the
 * state to the device (synchronising `stream`) and returns the saved step in
 * *step (may be NULL).  Both allocate host memory for one shard.
 * Errors: ZR_ERR_IO (file), ZR_ERR_MISMATCH (another partition or rank, or a
 * corrupt file), ZR_ERR_CUDA, ZR_ERR_INVALID_ARG. */
zr_status zr_state_save(const zr_plan* plan, const char* path, const float* master, const float* m,
                        const float* v, int64_t step, zr_stream_t stream);
zr_status zr_state_load(const zr_plan* plan, const char* path, float* master, float* m, float* v,
                        int64_t* step, zr_stream_t stream);

/* Elastic resume: writes to dst_path the shard of `target`'s rank under
 * `target`'s partition, built from src_paths[0..n_src), the complete set of
 * shards (rank r at index r) that another partition of the same tensors
 * saved (any W, either mode, same step).  Host only; reads each source
 * shard whole once.  A target with W = 1 and the flat mode yields the whole
 * fp32 state in declaration order.  Errors: ZR_ERR_IO, ZR_ERR_MISMATCH
 * (shards of other tensors, missing or out-of-order ranks, different steps,
 * corrupt payloads), ZR_ERR_INVALID_ARG. */
zr_status zr_state_reshard(const zr_plan* target, const char* const* src_paths, int32_t n_src,
                           const char* dst_path);

/* Gather to a whole model on save: from src_paths[0..n_src), the complete
 * set of shards (rank r at index r) of any partition of `plan`'s tensors
 * (`plan` supplies the shapes only; its W, rank and mode do not matter),
 * writes the master weights of all total_numel parameters in declaration
 * order -- tensor by tensor, each row-major, no pad -- to out_path as a raw
 * little-endian array: fp32 (ZR_EXPORT_F32) or bf16 rounded to nearest even
 * (ZR_EXPORT_BF16, the value the step writes into the all-gather buffer).
 * No header: the file is exactly total_numel * 4 or * 2 bytes.  Host only;
 * reads each shard whole once, holds the output in host memory and writes it
 * through a temporary file renamed into place; *n_written (may be NULL)
 * receives total_numel.  Errors as zr_state_reshard, and ZR_ERR_INVALID_ARG
 * for an unknown dtype. */
#define ZR_EXPORT_F32 0
#define ZR_EXPORT_BF16 1
zr_status zr_state_export_params(const zr_plan* plan, const char* const* src_paths, int32_t n_src,
                                 int32_t dtype, const char* out_path, int64_t* n_written);

/* ZeRO-3 (parameters sharded too): "Scaling training to thousands of GPUs"
 * (talk summary), section 11:24 ZeRO, and "CS336 lecture 8", section "ZeRO
 * levels": stage 3 keeps only this rank's slice of the bf16 parameters and
 * all-gathers each layer's full parameters just before the layer needs
 * them, a step ahead (prefetch), freeing them after use.
 *
 * zr_plan_set_param_layout selects where the step writes the bf16
 * parameters: ZR_PARAMS_GLOBAL (the default) -- param_out is the full
 * all-gather buffer (padded_numel elements, global layout); ZR_PARAMS_OWNED
 * -- param_out is this rank's shard, owned_numel elements in owned order
 * (the order of master / m / v).  It applies to every step call (zr_step,
 * zr_step_device_count, zr_step_bucket / zr_step_finish, zr_step_host,
 * zr_step_no_alloc; zr_step_host then copies the shard back in owned
 * order).  Changing it rebuilds the tile tables and, when a workspace is
 * bound, uploads them on `stream` and clears checked mode's status; work
 * queued on other streams that reads the tables must be ordered before it.
 * ZR_PARAMS_OWNED with gather targets set is ZR_ERR_UNSUPPORTED.
 *
 * zr_gather_params writes tensors first_tensor .. first_tensor + n_tensors
 * - 1 (declaration order), whole and in the global layout, to dst (bf16,
 * consecutive, row-major; 16-byte aligned), gathered from shard_ptrs[w] =
 * rank w's bf16 shard in owned order (W device pointers, local or mapped
 * from other GPUs, 16-byte aligned; NULL allowed for a rank that owns
 * nothing).  dst must not overlap any shard.
 * One kernel on `stream`: pieces of at most 16384 elements of one tensor
 * and one owner, plain 16-byte loads and stores where source and
 * destination share their alignment, 2-byte ones otherwise, with the
 * streaming (evict-first) cache hint; one CTA per piece when max_ctas <= 0,
 * else at most max_ctas CTAs looping over the pieces (for a prefetch that
 * should leave most SMs to the compute it overlaps).  Issue it on a side
 * stream a layer ahead to prefetch.  Errors: ZR_ERR_INVALID_ARG (range,
 * NULL), ZR_ERR_ALIGNMENT (dst), ZR_ERR_NO_WORKSPACE, ZR_ERR_CUDA. */
#define ZR_PARAMS_GLOBAL 0
#define ZR_PARAMS_OWNED 1
zr_status zr_plan_set_param_layout(zr_plan* plan, int32_t layout, zr_stream_t stream);
zr_status zr_gather_params(const zr_plan* plan, int32_t first_tensor, int32_t n_tensors,
                           const void* const* shard_ptrs, void* dst, int32_t max_ctas, zr_stream_t stream);

/* Checked mode: a stand-in for a memory sanitizer at run time.  The plan's
 * tile tables live in the caller's workspace, so a kernel that writes there
 * by mistake (a race on the workspace, a stray pointer) would send the next
 * step to wrong or out-of-bounds addresses.  The pages have no counterpart;
 * it follows from this library's caller-owned workspace.
 *
 * zr_plan_verify enqueues on `stream` one kernel that tests every tile of
 * both device tile tables against the invariants the planner guarantees
 * (length 1..2048, owned and output ranges inside the rank's owned count
 * and the output buffer, 16-byte vector flags only where the alignment
 * holds, bucket and index in range, each bucket-order tile at its own
 * index) and every entry of the ZeRO-3 gather piece table (length
 * 1..16384, owner and tensor in range, destination inside total_numel),
 * and compares an order-independent 64-bit hash of each table with the one
 * taken on the host when it was uploaded.  If anything fails, now or at an
 * earlier check, all three tables are overwritten with empty entries, so
 * the steps and gathers queued after it update and write nothing (their
 * results are then missing, not wrong); zr_plan_set_workspace re-uploads
 * the tables and clears the status.  Nothing waits on anything; a check is one small
 * launch reading 64 bytes per tile.
 * zr_plan_set_checked(plan, 1) makes every call that launches kernels
 * reading those tables (zr_step, zr_step_device_count, zr_step_bucket,
 * zr_step_finish, zr_step_host, zr_grad_sumsq, zr_debug_reduce,
 * zr_gather_params) run that check first on its stream; 0 (the default)
 * turns it off.  zr_step_no_alloc keeps its own copy
 * of the table and is not affected.
 * zr_plan_check_result synchronises `stream` and reads the status:
 * bad_tiles = entries that failed an invariant (all tables, counted at every
 * check since the workspace was bound), first_bad = the smallest failing
 * position (i for the bucket-order tile table, n_tiles + i for the
 * owned-order one, 2 n_tiles + i for the gather pieces) or -1,
 * hash_mismatch = bit 0 for the bucket-order table, bit 1 for the
 * owned-order one, bit 2 for the gather pieces, tables_emptied = 1 once a
 * failure has emptied them.
 * Errors: ZR_ERR_INVALID_ARG, ZR_ERR_NO_WORKSPACE, ZR_ERR_CUDA. */
typedef struct {
    uint64_t bad_tiles;
    int64_t first_bad;
    uint32_t hash_mismatch;
    uint32_t tables_emptied;
} zr_check_result;

zr_status zr_plan_set_checked(zr_plan* plan, int32_t enable);
zr_status zr_plan_verify(const zr_plan* plan, zr_stream_t stream);
zr_status zr_plan_check_result(const zr_plan* plan, zr_check_result* out, zr_stream_t stream);

/* Size of the library-owned scratch array used by zr_step_no_alloc. */
#define ZR_NO_ALLOC_SCRATCH_BYTES (4u << 20)

/* zr_step for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call; it exists for callers such as a plug-in inside a
 * host framework whose allocator owns all of the GPU's memory (a caching
 * allocator that has reserved it, or a framework that forbids outside
 * cudaMalloc), or a latency-critical loop that must not call cudaMalloc
 * because it can synchronise the device.  Such callers have their inputs
 * and outputs but cannot give the plan a workspace.
 *
 * Same arguments and results as zr_step, plus d_sumsq_partials (clipping
 * only; otherwise may be NULL): the device array of world_size doubles that
 * zr_plan_set_sumsq_partials would bind -- other ranks' S_w in, this rank's
 * entry written.  No workspace needs to be bound; the call makes no
 * cudaMalloc or cudaFree and calls no allocating routine.  It runs zr_step's
 * kernels in zr_step's order, so master, m, v, param_out and S_r are
 * bit-identical to zr_step's.
 *
 * Scratch (the tile table and, with clipping, one double per tile, one per
 * group of 1024 tiles and a counter) lives in a file-scope device
 * array of ZR_NO_ALLOC_SCRATCH_BYTES (4 MiB) that every GPU that loads the
 * library holds until the process exits.  The plan needs 32 bytes per tile,
 * plus about 8 more per tile with clipping, plus about 1 KB: up to about
 * 131,000 tiles (about 104,800 with clipping).  A tile covers up to 2048
 * owned elements, so a shard of up to about 268 M owned elements fits
 * (about 214 M with clipping).  A larger plan gets ZR_ERR_UNSUPPORTED before
 * anything is launched: use zr_step with a workspace instead.  With
 * clipping, the second pass reads the gradients again instead of keeping an
 * fp32 copy of the averaged gradient (the same values: the fold is
 * deterministic).
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it for the life of the process; make
 * that first call before any stream capture.  cudaDeviceReset is not
 * supported: after it the cached address, and the record of which table
 * the array holds, would be stale.
 *
 * The tile table is copied from the plan's host memory (an asynchronous
 * copy on `stream` from pageable memory) when the array does not already
 * hold this plan's current table: on the plan's first call on the device,
 * after another plan's call on that device, and after
 * zr_plan_set_param_layout rebuilt the plan's tables.  A loop that steps one
 * plan copies it once; its later calls enqueue only kernels (and, with
 * clipping, a device-side memset of the counter, which must start at
 * zero).  Every call, on every plan, uses the same array and leaves its
 * contents behind.  Calls whose work overlaps on the GPU (different streams
 * without ordering between them) race on the array and give wrong results.
 * Errors: as zr_step, plus ZR_ERR_UNSUPPORTED (plan too large for the array,
 * or the current device is not compute capability 10.x). */
zr_status zr_step_no_alloc(const zr_plan* plan, const void* const* grad_ptrs, float* master, float* m,
                           float* v, void* param_out, double* d_sumsq_partials, int64_t step,
                           zr_stream_t stream);

void zr_plan_destroy(zr_plan* plan);

const char* zr_status_string(zr_status status);

#ifdef __cplusplus
}
#endif

#endif /* ZR_H_ */
