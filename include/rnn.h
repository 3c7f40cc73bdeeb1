/*
 * rnn.h - reciprocal nearest-neighbour matching on B200 (sm_100a).
 *
 * A C ABI over hand-written CUDA kernels.  The operations are those of dense
 * descriptor matching in MASt3R:
 *
 *   descriptors   D1 in R^{H1 x W1 x d}, D2 in R^{H2 x W2 x d}, one d-vector
 *                 per pixel (cv-learn.com "MASt3R" note, section "Method and
 *                 architecture", matching head).  Stored channel-last and
 *                 row-major as fp16 or bf16: element (y, x, c) of a map is at
 *                 offset (y*W + x)*d + c.  Pixel index p = y*W + x.
 *   score         s(i, j) = sum_c D1[i][c] * D2[j][c], accumulated in fp32.
 *   NN2(i)        the lowest j with the largest s(i, j); NN1(j) likewise over
 *                 i.  (The pages name nearest neighbours without a metric or a
 *                 tie rule; the descriptors are unit vectors, so the largest
 *                 dot product is also the smallest Euclidean distance.)
 *   M             {(i, j) : j = NN2(i) and i = NN1(j)}, the reciprocal set
 *                 (same note, paragraph "Fast reciprocal matching (FRM)").
 *
 * Conventions for every entry point:
 *   - Every array argument is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or synchronises, and every result
 *     (including counts) is ordered on `stream` like a kernel's output.
 *   - Descriptor pointers must be 16-byte aligned and d a multiple of 8
 *     (RNN_EALIGN otherwise); 8 <= d <= 256 (RNN_EUNSUPPORTED above).
 *   - Inputs must be finite and their scores finite in fp32; NaN or Inf gives
 *     undefined matches (but no out-of-bounds access).
 *   - Argument errors are returned before anything is launched.  A launch
 *     failure returns RNN_ECUDA.  The kernels' internal waits are bounded;
 *     if one runs out the kernel stops early and records it in the workspace,
 *     which rnn_workspace_status() reports as RNN_ETIMEOUT.
 *   - Calls that share a workspace must not overlap on the device.
 *   - The GPU must be sm_100 (B200); otherwise RNN_EUNSUPPORTED.
 *   - Pairs are written as int32 (i, j) = (image-1 pixel, image-2 pixel).
 */
#ifndef RNN_H
#define RNN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *rnn_stream_t;

typedef enum rnn_status {
  RNN_OK = 0,
  RNN_EINVAL = 1,       /* null pointer, non-positive size, bad stride or count */
  RNN_EALIGN = 2,       /* d not a multiple of 8, or a pointer not 16-byte aligned */
  RNN_ECAPACITY = 3,    /* output capacity below the guaranteed maximum */
  RNN_ECUDA = 4,        /* a CUDA runtime or driver call failed */
  RNN_ETIMEOUT = 5,     /* a kernel's bounded wait ran out (see rnn_workspace_status) */
  RNN_EUNSUPPORTED = 6, /* d > 256, too many pairs in a batch, or not an sm_100 GPU */
  RNN_EWORKSPACE = 7    /* workspace missing, too small or not 256-byte aligned */
} rnn_status;

typedef enum rnn_dtype { RNN_F16 = 0, RNN_BF16 = 1 } rnn_dtype;

/*
 * Meaning of "nearest" (the *_ex entry points; the others use RNN_DOT):
 *   RNN_DOT  the largest dot product s(i, j) = sum_c D1[i][c] * D2[j][c];
 *            for unit descriptors, as the matching head emits, this is the
 *            nearest neighbour in Euclidean distance (cv-learn.com "MASt3R"
 *            note, section "Method and architecture").
 *   RNN_L2   the smallest Euclidean distance |D1_i - D2_j|, which is what the
 *            brute-force matcher of the quoted fast_reciprocal_NNs computes
 *            (all distances, the smallest kept; staskaer.github.io
 *            DUSt3R/MASt3R blog, MASt3R matching section).
 * Ties go to the lowest index under either metric.
 */
typedef enum rnn_metric { RNN_DOT = 0, RNN_L2 = 1 } rnn_metric;

/* Largest batch of the batched FRM entry point. */
#define RNN_MAX_BATCH 1024

/* Human-readable name of a status. */
const char *rnn_status_string(rnn_status s);

/* Version of this ABI (incremented on any signature change). */
int rnn_abi_version(void);

/*
 * Device-side status of the most recent call that used `workspace`:
 * synchronises `stream`, then returns RNN_ETIMEOUT if a kernel of that call
 * gave up on a bounded wait, else RNN_OK (RNN_ECUDA if the copy fails).
 */
rnn_status rnn_workspace_status(const void *workspace, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Nearest neighbours of a set of queries (the NN1 / NN2 operator).
 *
 * NN2(D1_i) is the pixel of image 2 whose descriptor best matches D1_i, and
 * NN1 the same from image 2 into image 1 (cv-learn.com "MASt3R" note,
 * paragraph "Fast reciprocal matching (FRM)"; the staskaer.github.io
 * DUSt3R/MASt3R blog, MASt3R matching section, where the quoted
 * fast_reciprocal_NNs calls it on the active seeds at every half-step).
 * Best = largest dot product, lowest index among equal scores.
 *
 *   Q          [nq][d] query descriptors.
 *   X          [nx][d] candidate descriptors.
 *   idx_out    [nq] int32: NN of each query among the rows of X (lowest index
 *              among equal largest scores).
 *   score_out  [nq] float: that largest score (may be NULL).
 *   workspace  at least rnn_nn_workspace_size(nq) bytes, 256-byte aligned.
 * nq may be 0 (then Q and idx_out may be NULL and only the workspace status is
 * reset); nx must be >= 1.
 */
size_t rnn_nn_workspace_size(int64_t nq);
rnn_status rnn_nn_argmax(const void *Q, int64_t nq, const void *X, int64_t nx, int d,
                         rnn_dtype dtype, int32_t *idx_out, float *score_out, void *workspace,
                         size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Exhaustive reciprocal set M between two maps (cv-learn.com "MASt3R" note,
 * paragraph "Fast reciprocal matching (FRM)": the O(W^2 H^2) mutual-NN set).
 *
 *   pairs_out  [cap][2] int32: M in increasing i.  cap >= min(H1*W1, H2*W2)
 *              (RNN_ECAPACITY otherwise), which no M can exceed.
 *   count_out  [1] int32: |M|.
 *   rowarg_out [H1*W1] NN2 of every D1 pixel, rowmax_out its score,
 *   colarg_out [H2*W2] NN1 of every D2 pixel, colmax_out its score;
 *              each of these four may be NULL.
 *   workspace  at least rnn_mnn_workspace_size(H1, W1, H2, W2, d) bytes,
 *              256-byte aligned.  For d <= 64 it holds copies of both maps
 *              made by the call (rows zero-padded to the K-block, then 2048
 *              NaN rows past the last pixel), which one pass of the fused
 *              kernel reduces by rows and by columns; larger d keeps the
 *              rows as given (two sweeps, one per direction).
 */
size_t rnn_mnn_workspace_size(int H1, int W1, int H2, int W2, int d);
rnn_status rnn_mnn_exhaustive(const void *D1, int H1, int W1, const void *D2, int H2, int W2,
                              int d, rnn_dtype dtype, int32_t *pairs_out, int64_t cap,
                              int32_t *count_out, int32_t *rowarg_out, float *rowmax_out,
                              int32_t *colarg_out, float *colmax_out, void *workspace,
                              size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Fast Reciprocal Matching (cv-learn.com "MASt3R" note, paragraph "Fast
 * reciprocal matching (FRM)"; loop semantics of the fast_reciprocal_NNs
 * function quoted in the staskaer.github.io DUSt3R/MASt3R blog, MASt3R
 * matching section):
 *
 *   seeds  u on image 1 at rows y = S/2, S/2+S, ... < H1 and columns
 *          x = S/2, S/2+S, ... < W1 (S = seed_stride, integer halving),
 *          ascending; U = seeds, V = -1, U_old = U, V_old = V, all active.
 *   loop   for t = 1 .. max_iter, while some seed is active:
 *            V = NN2(U) for the active seeds; deactivate those with V == V_old;
 *            U = NN1(V) for the still-active seeds; deactivate those with
 *            U == U_old; stop after iteration max_iter; else U_old = U,
 *            V_old = V.
 *   output the (U, V) of the seeds that are no longer active, unique, sorted
 *          by U.  Every output pair is in M.
 *
 * The whole loop runs on the device: 4*max_iter + 4 kernel launches (2 more
 * when d needs padded copies), no host synchronisation.
 *
 *   seed_stride >= 1, max_iter >= 1 (RNN_EINVAL otherwise).
 *   pairs_out   [cap][2] int32, cap >= rnn_frm_max_pairs(...).
 *   count_out   [1] int32.
 *   seed_state_out  (may be NULL) [k][4] int32 per seed: final U, final V,
 *               number of NN queries made for it, 1 if converged else 0.
 *   workspace   at least rnn_frm_workspace_size(1, H1, W1, H2, W2, d, seed_stride)
 *               bytes, 256-byte aligned (it holds zero-padded copies of the
 *               maps when d is not a whole number of K-blocks).
 */
int64_t rnn_frm_num_seeds(int H1, int W1, int seed_stride);
int64_t rnn_frm_max_pairs(int H1, int W1, int H2, int W2, int seed_stride);
size_t rnn_frm_workspace_size(int B, int H1, int W1, int H2, int W2, int d, int seed_stride);
rnn_status rnn_frm_match(const void *D1, int H1, int W1, const void *D2, int H2, int W2, int d,
                         rnn_dtype dtype, int seed_stride, int max_iter, int32_t *pairs_out,
                         int64_t cap, int32_t *count_out, int32_t *seed_state_out,
                         void *workspace, size_t ws_bytes, rnn_stream_t stream);

/*
 * FRM over B independent pairs in one launch sequence.  Pair b reads
 * D1 + b*d1_batch_stride and D2 + b*d2_batch_stride (strides in elements,
 * multiples of 8, at least H*W*d) and writes pairs_out + b*cap*2,
 * count_out[b] and seed_state_out + b*k*4.  1 <= B <= RNN_MAX_BATCH.
 */
rnn_status rnn_frm_match_batched(int B, const void *D1, int64_t d1_batch_stride, const void *D2,
                                 int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                                 rnn_dtype dtype, int seed_stride, int max_iter,
                                 int32_t *pairs_out, int64_t cap, int32_t *count_out,
                                 int32_t *seed_state_out, void *workspace, size_t ws_bytes,
                                 rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * The same operations with every option of the quoted fast_reciprocal_NNs
 * (staskaer.github.io DUSt3R/MASt3R blog, MASt3R matching section) and the
 * metric.  The entry points above are these with RNN_DOT, the grid seeds,
 * no pixel tolerance and no basin.
 *
 * rnn_nn_argmax_ex / rnn_mnn_exhaustive_ex: as rnn_nn_argmax /
 * rnn_mnn_exhaustive.  With RNN_L2 the scores written (score_out, rowmax_out,
 * colmax_out) are squared distances |q - x|^2 of the chosen neighbours.
 * Their workspace sizes depend on the metric.  The Euclidean metric keeps
 * augmented copies of the maps in it: for rnn_nn_argmax_ex (and the
 * exhaustive set with d > 56) rows [x, -|x|^2/2 in three 16-bit parts] and
 * [q, 1, 1, 1], whose dot product q.x - |x|^2/2 the tensor cores maximise;
 * for the exhaustive set with d <= 56 rows [q, 1, 1, 1, -|q|^2/2] of image 1
 * and [x, -|x|^2/2, 1, 1, 1] of image 2, whose dot product -|q - x|^2/2 is
 * maximised over rows and over columns in one pass.
 *
 * rnn_frm_match_ex: FRM over B pairs (as rnn_frm_match_batched) with
 *   init_xy1     NULL: seeds on the grid of stride seed_stride (>= 1).
 *                Else device int32 [B][n_init] start pixels y*W1 + x of each
 *                pair; they are made unique and ascending (starts outside
 *                the image are dropped), and seed_stride is not used.  The
 *                quoted function runs given starts for one iteration
 *                (max_iter = 1); any max_iter >= 1 is accepted.
 *   pixel_tol    0: a seed is output when it is no longer active, as (U, V).
 *                > 0 (only with init_xy1, else RNN_EINVAL): a seed is output
 *                when its last move, from U_old to U, is shorter than
 *                pixel_tol pixels (Euclidean distance of the row/column
 *                positions), as (U_old, V): with one iteration, the start
 *                pixel and its match.
 *   basin_out    NULL, or device int32 [B][H1*W1 + 1]: basin mode.  The first
 *                half-step then deactivates no seed, and after the second,
 *                basin[U_old] = U for every seed it served; entries never
 *                written are -1 (the last entry always).  The output pairs
 *                are the same as without basin mode.
 *   pairs_out    [B][cap][2], cap >= min(k, H2*W2), or cap >= k with a pixel
 *                tolerance; k = n_init with given starts, else the grid size.
 *   seed_state_out  (may be NULL) [B][k][4] per seed slot: final U, final V,
 *                queries made, 1 if output; slots past a pair's unique starts
 *                hold -1, -1, 0, 0.
 * rnn_frm_workspace_size_ex takes n_init = the starts per pair, or -1 for the
 * grid of stride seed_stride.
 * 4 + 4*max_iter kernel launches, plus 2 (padded copies, dot metric with
 * d = 8, 24, 40, ...) or 4 (Euclidean metric) for the row copies, plus 2 with
 * given starts.
 */
size_t rnn_nn_workspace_size_ex(int64_t nq, int64_t nx, int d, rnn_metric metric);
rnn_status rnn_nn_argmax_ex(const void *Q, int64_t nq, const void *X, int64_t nx, int d,
                            rnn_dtype dtype, rnn_metric metric, int32_t *idx_out,
                            float *score_out, void *workspace, size_t ws_bytes,
                            rnn_stream_t stream);
size_t rnn_mnn_workspace_size_ex(int H1, int W1, int H2, int W2, int d, rnn_metric metric);
rnn_status rnn_mnn_exhaustive_ex(const void *D1, int H1, int W1, const void *D2, int H2, int W2,
                                 int d, rnn_dtype dtype, rnn_metric metric, int32_t *pairs_out,
                                 int64_t cap, int32_t *count_out, int32_t *rowarg_out,
                                 float *rowmax_out, int32_t *colarg_out, float *colmax_out,
                                 void *workspace, size_t ws_bytes, rnn_stream_t stream);
size_t rnn_frm_workspace_size_ex(int B, int H1, int W1, int H2, int W2, int d,
                                 rnn_metric metric, int seed_stride, int64_t n_init);
rnn_status rnn_frm_match_ex(int B, const void *D1, int64_t d1_batch_stride, const void *D2,
                            int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                            rnn_dtype dtype, rnn_metric metric, const int32_t *init_xy1,
                            int64_t n_init, int seed_stride, int max_iter, float pixel_tol,
                            int32_t *pairs_out, int64_t cap, int32_t *count_out,
                            int32_t *seed_state_out, int32_t *basin_out, void *workspace,
                            size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * FRM graph plans.  rnn_frm_graph_create records one rnn_frm_match_ex call
 * (same arguments, minus the stream) as a CUDA graph and instantiates it;
 * rnn_frm_graph_launch replays it on a stream.  Iterations 2..max_iter sit
 * in conditional nodes: the last step kernel of each iteration enables the
 * next one only while some seed of some pair is still active, so iterations
 * after convergence launch nothing (the results are those of the call, bit
 * for bit: an iteration with no active seed changes no state).
 *   The plan holds the device pointers it was given (maps, starts, outputs,
 *   workspace): every launch reads the maps' current contents and rewrites
 *   the outputs; the buffers must outlive the plan, and launches of one plan
 *   must not overlap (they share the workspace).  max_iter <= 64
 *   (RNN_EUNSUPPORTED).  The argument checks and errors are those of
 *   rnn_frm_match_ex, plus RNN_ECUDA if graph creation fails.  The status
 *   word of the workspace (rnn_workspace_status) reports a launch's errors.
 *   *graph_out is owned by the caller: release it with rnn_frm_graph_destroy
 *   (NULL is accepted).
 * An FRM call (rnn_frm_match*, rnn_c2f_match) that the caller itself records
 * into a CUDA graph (stream capture) records its iterations 2..max_iter in
 * conditional nodes of that graph the same way, when max_iter <= 64 and the
 * calling thread has made an FRM call outside a capture before: that call
 * creates the per-thread stream the iteration bodies are recorded on, since
 * no stream is created inside a capture.  Otherwise every iteration is
 * recorded.  Either way a replay gives the call's results.
 */
typedef struct rnn_frm_graph *rnn_frm_graph_t;
rnn_status rnn_frm_graph_create(int B, const void *D1, int64_t d1_batch_stride, const void *D2,
                                int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                                rnn_dtype dtype, rnn_metric metric, const int32_t *init_xy1,
                                int64_t n_init, int seed_stride, int max_iter, float pixel_tol,
                                int32_t *pairs_out, int64_t cap, int32_t *count_out,
                                int32_t *seed_state_out, int32_t *basin_out, void *workspace,
                                size_t ws_bytes, rnn_frm_graph_t *graph_out);
rnn_status rnn_frm_graph_launch(rnn_frm_graph_t graph, rnn_stream_t stream);
void rnn_frm_graph_destroy(rnn_frm_graph_t graph);

/* ------------------------------------------------------------------------
 * The reciprocal set from NN arrays computed elsewhere (cv-learn.com "MASt3R"
 * note, paragraph "Fast reciprocal matching (FRM)": M = {(i, j) | j = NN2(i)
 * and i = NN1(j)}), e.g. when the rows of both maps are split over several
 * GPUs, each computes NN2 / NN1 for its rows, and the arrays are gathered.
 *
 *   rowarg     device int32 [n1]: NN2 of every image-1 pixel.
 *   colarg     device int32 [n2]: NN1 of every image-2 pixel.
 *   pairs_out  [cap][2] int32: (i, rowarg[i]) for every i with
 *              colarg[rowarg[i]] == i, in increasing i; cap >= min(n1, n2).
 *              Indices outside [0, n2) in rowarg are never mutual.
 *   count_out  [1] int32.
 *   workspace  at least rnn_mnn_mutual_workspace_size(n1) bytes.
 * 2 kernel launches (and one memset of the workspace header).
 */
size_t rnn_mnn_mutual_workspace_size(int64_t n1);
rnn_status rnn_mnn_mutual(const int32_t *rowarg, int64_t n1, const int32_t *colarg, int64_t n2,
                          int32_t *pairs_out, int64_t cap, int32_t *count_out, void *workspace,
                          size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Coarse-to-fine matching (cv-learn.com "MASt3R" note, paragraph
 * "Coarse-to-fine matching": high-resolution images are matched coarsely
 * first, the coarse matches guide the matching of enumerated local crops,
 * and the fine matches are mapped back to full resolution; the
 * staskaer.github.io DUSt3R/MASt3R blog describes the same step as matching
 * again block by block at full resolution).  The pages give no formulas for
 * the crops; these integer rules are this library's:
 *
 *   coarse     M of the coarse maps C1 [Hc1][Wc1][dc], C2 [Hc2][Wc2][dc]
 *              (rnn_mnn_exhaustive_ex with `metric`).
 *   pixel      coarse pixel (yc, xc) of an Hc x Wc map stands for the
 *              full-resolution pixel (floor((2yc+1)H/(2Hc)), floor((2xc+1)W/(2Wc))).
 *   crops      ch = min(crop_h, H1, H2), cw = min(crop_w, W1, W2); image 1 is
 *              covered by ceil(H1/ch) x ceil(W1/cw) crops, row-major, at
 *              origins floor(a*(L-c)/(n-1)) along each axis (0 when n = 1).
 *              At most RNN_MAX_BATCH crops (RNN_EUNSUPPORTED).
 *   pairing    crop b holds the coarse pairs whose image-1 pixel lies inside
 *              it; with at least max(min_coarse, 1) of them it is on, and its
 *              image-2 crop is centred on the floor of the mean of their
 *              image-2 pixels, clamped into image 2.
 *   fine       FRM (grid seeds of stride seed_stride inside the crop,
 *              max_iter) between the windows of F1 [H1][W1][d] and F2
 *              [H2][W2][d] of every crop pair that is on, batched.
 *   output     each pair mapped back by its crops' origins; where crops
 *              overlap, the lowest crop index that outputs an image-1 pixel
 *              gives its pair; pairs_out [cap][2] sorted by the image-1
 *              pixel, count_out [1].  cap >= rnn_c2f_max_pairs(...).
 *   crops_out  NULL or device int32 [ncrops][6]: y0_1, x0_1, y0_2, x0_2,
 *              coarse pairs inside, on.
 * All four maps share dtype; C1/C2 and F1/F2 follow the descriptor rules
 * (16-byte aligned, dc and d multiples of 8).  rnn_workspace_status() on the
 * workspace reports a timed-out wait of any part.  No host synchronisation;
 * 15 + 4*max_iter kernel launches, plus the row copies: 2 when dc needs
 * padding (dc = 8, 24, 40, ...), and with RNN_L2 4 for the coarse and 4 for
 * the fine Euclidean forms.
 */
int rnn_c2f_num_crops(int H1, int W1, int H2, int W2, int crop_h, int crop_w);
int64_t rnn_c2f_max_pairs(int H1, int W1, int H2, int W2, int crop_h, int crop_w,
                          int seed_stride);
size_t rnn_c2f_workspace_size(int Hc1, int Wc1, int Hc2, int Wc2, int dc, int H1, int W1,
                              int H2, int W2, int d, rnn_metric metric, int crop_h, int crop_w,
                              int seed_stride);
rnn_status rnn_c2f_match(const void *C1, int Hc1, int Wc1, const void *C2, int Hc2, int Wc2,
                         int dc, const void *F1, int H1, int W1, const void *F2, int H2, int W2,
                         int d, rnn_dtype dtype, rnn_metric metric, int crop_h, int crop_w,
                         int seed_stride, int max_iter, int min_coarse, int32_t *pairs_out,
                         int64_t cap, int32_t *count_out, int32_t *crops_out, void *workspace,
                         size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * 3-D points.  MASt3R picks the NN function of reciprocal matching by the
 * dimension of its input, and matches 3-D points (its point maps) with K-d
 * trees (MASt3R paper text quoted in the staskaer.github.io DUSt3R/MASt3R
 * blog, MASt3R matching section).  These entry points compute the same
 * thing: the exact nearest point in Euclidean distance, lowest index on
 * ties, and with it the reciprocal set and FRM on point maps.
 *
 *   points     fp32 [n][3] (x, y, z), 4-byte aligned DEVICE pointers (RNN_EALIGN
 *              otherwise); point maps [H][W][3], pixel p = y*W + x.
 *   distances  squared Euclidean distances, computed in fp32 as
 *              fma(dz, dz, fma(dy, dy, dx*dx)) with d = q - x; the NN is the
 *              lowest index with the smallest such value.  On coordinates that
 *              are multiples of 2^-6 within [-16, 16] every such value is
 *              exact (each partial result is a multiple of 2^-12 below 2^12).
 *   sizes      at most 2^28 points per set (RNN_EUNSUPPORTED above).
 *   inputs     finite; NaN or Inf gives undefined matches (but valid indices
 *              and no out-of-bounds access).
 *   time       a uniform grid over each set's bounding box (cells of about
 *              two point spacings on a surface through the box): a query
 *              visits a few cells on point maps of surfaces; a query far from
 *              the set, or a set with most points in a few cells, costs up to
 *              a pass over every point.
 *
 * rnn_pts_nn: NN of each of the nq query points among the nx >= 1 points of
 *   X.  idx_out [nq] int32, dist2_out [nq] float (may be NULL).  nq may be 0.
 *   7 kernel launches (6 when nq = 0).
 * rnn_pts_mnn: the reciprocal set between two point maps; outputs as
 *   rnn_mnn_exhaustive, with squared distances in rowd2_out / cold2_out.
 *   9 kernel launches.
 * rnn_pts_frm_match: FRM over B pairs of point maps with every option of
 *   rnn_frm_match_ex (batch strides in floats, at least 3*H*W; init_xy1,
 *   n_init, pixel_tol, basin_out, cap and seed_state_out as there).
 *   rnn_pts_frm_workspace_size takes n_init = starts per pair, or -1 for the
 *   grid of stride seed_stride.  10 + 2*max_iter kernel launches (2 more with
 *   given starts).
 */
size_t rnn_pts_nn_workspace_size(int64_t nq, int64_t nx);
rnn_status rnn_pts_nn(const float *Q, int64_t nq, const float *X, int64_t nx, int32_t *idx_out,
                      float *dist2_out, void *workspace, size_t ws_bytes, rnn_stream_t stream);
size_t rnn_pts_mnn_workspace_size(int H1, int W1, int H2, int W2);
rnn_status rnn_pts_mnn(const float *P1, int H1, int W1, const float *P2, int H2, int W2,
                       int32_t *pairs_out, int64_t cap, int32_t *count_out, int32_t *rowarg_out,
                       float *rowd2_out, int32_t *colarg_out, float *cold2_out, void *workspace,
                       size_t ws_bytes, rnn_stream_t stream);
size_t rnn_pts_frm_workspace_size(int B, int H1, int W1, int H2, int W2, int seed_stride,
                                  int64_t n_init);
rnn_status rnn_pts_frm_match(int B, const float *P1, int64_t p1_batch_stride, const float *P2,
                             int64_t p2_batch_stride, int H1, int W1, int H2, int W2,
                             const int32_t *init_xy1, int64_t n_init, int seed_stride,
                             int max_iter, float pixel_tol, int32_t *pairs_out, int64_t cap,
                             int32_t *count_out, int32_t *seed_state_out, int32_t *basin_out,
                             void *workspace, size_t ws_bytes, rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Nearest neighbours without any allocation.  (The matching method itself
 * has no counterpart of this: it exists for callers, not for the algorithm.)
 *
 * Same computation, arguments, results and errors as rnn_nn_argmax, minus the
 * workspace: its scratch lives in a fixed array inside the library, which
 * every GPU that loads the library keeps for the life of the process
 * (256 + 8 * RNN_NN_NOALLOC_MAX_QUERIES bytes, about 512 KB).  It is meant for
 * callers that cannot allocate device memory themselves: a plugin whose host
 * framework owns all device buffers, or a latency-bound loop in which
 * cudaMalloc/cudaFree would synchronise the device.  The function itself calls
 * no allocator.
 *
 *   nq > RNN_NN_NOALLOC_MAX_QUERIES  -> RNN_EUNSUPPORTED (nothing launched).
 *   The call looks up the array's device address with the caller's device
 *   current (on a stream that is being captured it reuses the address the
 *   device's last other call found, so make the first call on a device before
 *   any stream capture).
 *   All calls share the one array, which keeps the last call's contents (each
 *   call clears what must start at zero): calls that overlap on the GPU, on
 *   any streams, race and give undefined results.  Serialise them.
 *   rnn_workspace_status() does not apply: rnn_nn_argmax_noalloc_status()
 *   reads the array's status word instead.
 */
#define RNN_NN_NOALLOC_MAX_QUERIES 65536
rnn_status rnn_nn_argmax_noalloc(const void *Q, int64_t nq, const void *X, int64_t nx, int d,
                                 rnn_dtype dtype, int32_t *idx_out, float *score_out,
                                 rnn_stream_t stream);

/* Status of the last rnn_nn_argmax_noalloc call on the current device:
 * RNN_ETIMEOUT if one of its bounded device-side waits ran out (its indices
 * are then undefined, though in range), else RNN_OK.  Reads the status word
 * of the shared array (4 bytes to the host) and synchronises `stream`; it
 * allocates nothing.  Like the call itself, this has no counterpart on the
 * source pages.
 *   RNN_ECUDA  -> the copy or the synchronisation failed. */
rnn_status rnn_nn_argmax_noalloc_status(rnn_stream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics for benchmarking (no effect on results).
 *
 * rnn_launch_count: number of kernels this library has launched in this
 *   process (all entry points, all devices).  Kernels that an FRM call records
 *   into a graph (a graph plan, or a caller's capture) are not counted, nor
 *   are replays, and such recordings do not use the timer below; the other
 *   entry points' kernels recorded in a caller's capture count when recorded.
 * rnn_set_kernel_timer: while set, every launch of the fused
 *   similarity+argmax kernel is bracketed by cudaEventRecord(start_events[i])
 *   and cudaEventRecord(stop_events[i]) on the launch stream, with
 *   i = (*recorded)++ for i < capacity (launches past capacity are still
 *   counted).  The events (cudaEvent_t, created by the caller with timing
 *   enabled) and the host counter stay owned by the caller; pass NULL
 *   pointers or capacity 0 to switch the timer off.  The setting is global to
 *   the process and not thread-safe against concurrent calls.
 */
uint64_t rnn_launch_count(void);
void rnn_set_kernel_timer(void *const *start_events, void *const *stop_events, int capacity,
                          int *recorded);

/*
 * Failure-detection test hook (no use in production).  While `on` is
 * nonzero, every launch of the fused similarity+argmax kernel loads no
 * candidate tile, so the bounded wait of its MMA warps on the first tile runs
 * out after `wait_limit_ns` (0: the default of 1 s); the kernel then stops
 * all its warps, frees tensor memory and returns, and the call's workspace
 * status reads RNN_ETIMEOUT (rnn_workspace_status).  Results of those calls
 * are undefined but every index written is in range.  Nothing faults, traps
 * or hangs; later calls with the hook off are unaffected.  Global to the
 * process, not thread-safe against concurrent calls.
 */
void rnn_test_stall_loads(int on, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* RNN_H */
