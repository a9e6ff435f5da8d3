"""GPU parity of the codec, skinny GEMM and decode-attention kernels against
the fp64 oracle, through the C ABI (include/qad.h) via the thin binding.

Tolerances (the method's own):
* codec: bit-exact;
* GEMM: |y - y_ref| <= 1e-3 * sum_k |w x| per output;
* attention: per element |o - o_ref| <= 2e-3 * sum_t p_t |v_t| plus half a
  bf16 ulp of o_ref (the output's defined bf16 rounding point), and per
  (row, head) ||o - bf16(o_ref)|| <= 2e-3 ||o_ref||.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import SEED

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return q


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


# ------------------------------------------------------------------ codec

def test_q4k_unpack_bit_exact(q, orc):
    W = synth.q4k_matrix_np(SEED, 70, 64, 2048)
    nb = W.size // 144
    qq, sc, m, d, dmin = [t.cpu().numpy() for t in q.q4k_unpack(torch.from_numpy(W).cuda(), nb)]
    blocks = W.reshape(-1, 144)
    for b in range(nb):
        oq, osc, om, od, odm = orc.q4k_decode(blocks[b])
        assert np.array_equal(qq[b], oq) and np.array_equal(sc[b], osc) and np.array_equal(m[b], om)
        assert (int(d[b]) & 0xFFFF) == od and (int(dmin[b]) & 0xFFFF) == odm


def test_q6k_unpack_bit_exact(q, orc):
    W = synth.q6k_matrix_np(SEED, 71, 32, 2048)
    g = np.random.default_rng(1)
    W.reshape(-1, 210)[:, 192:208] = g.integers(0, 256, (W.size // 210, 16), dtype=np.uint8)  # signed scales too
    nb = W.size // 210
    qq, sc, d = [t.cpu().numpy() for t in q.q6k_unpack(torch.from_numpy(W).cuda(), nb)]
    blocks = W.reshape(-1, 210)
    for b in range(nb):
        oq, osc, od = orc.q6k_decode(blocks[b])
        assert np.array_equal(qq[b], oq) and np.array_equal(sc[b], osc) and (int(d[b]) & 0xFFFF) == od


def test_q6k_pack_layout(q, orc):
    """Packed layout: plane A = the first 208 bytes of every block, plane D = d
    (rows padded with zeros to a multiple of 8 blocks); byte-exact."""
    for N, K in [(7, 768), (33, 17408), (1, 2304)]:
        W = synth.q6k_matrix_np(SEED, 72 + N, N, K)
        nb = K // 256
        nb8 = (nb + 7) // 8 * 8
        P = q.q6k_pack(torch.from_numpy(W).cuda(), N, K).cpu().numpy()
        assert P.size == N * nb * 208 + N * nb8 * 2 == q.q6k_packed_bytes(N, K)
        blocks = W.reshape(N, nb, 210)
        assert np.array_equal(P[:N * nb * 208].reshape(N, nb, 208), blocks[:, :, :208])
        D = P[N * nb * 208:].view(np.uint16).reshape(N, nb8)
        for n in range(N):
            for b in range(nb):
                assert D[n, b] == orc.q6k_decode(blocks[n, b])[2]
        assert (D[:, nb:] == 0).all()


# ------------------------------------------------------------------ GEMM

GEMM_CASES = [
    (4, 256, 1024, 1),     # the small single-matrix case: N=256, K=1024, one row
    (4, 37, 768, 5),       # ragged N (not a tile multiple), 3 blocks per row
    (4, 300, 2560, 12),    # 12 rows, many tiles
    (4, 64, 256, 16),      # maximum rows, one block per row
    (4, 1, 512, 9),        # a single output row
    (4, 1000, 5120, 8),    # largest one-n-tile row count
    (6, 37, 768, 3),       # Q6_K: odd block count -> rows alternate 4-byte alignment
    (6, 130, 4352, 12),
    (6, 33, 256, 16),
    (6, 5, 17408, 2),      # the down-projection depth
]


def _gemm(q, fmt, W, N, K, X, M, accumulate=False, Y0=None):
    Wd = torch.from_numpy(W).cuda()
    if fmt == 6:
        Wd = q.q6k_pack(Wd, N, K)
    Xd = _to_dev_bf16(X)
    Y = torch.zeros(M, N, device="cuda") if Y0 is None else Y0.clone()
    fn = q.q4k_gemm if fmt == 4 else q.q6k_gemm
    fn(Wd, N, K, Xd, M, Y, accumulate=accumulate)
    torch.cuda.synchronize()
    return Y.cpu().double().numpy()


@pytest.mark.parametrize("fmt,N,K,M", GEMM_CASES)
def test_gemm_parity(q, orc, fmt, N, K, M):
    W = (synth.q4k_matrix_np if fmt == 4 else synth.q6k_matrix_np)(SEED, 80 + N, N, K)
    X = synth.bf16_normal_np(SEED, 80 + M, (M, K))
    Yr, A = orc.gemm(fmt, W, N, K, X)
    Y = _gemm(q, fmt, W, N, K, X, M)
    ratio = np.abs(Y - Yr) / (1e-3 * A + 1e-30)
    assert ratio.max() <= 1.0, f"max err / tol = {ratio.max():.3g}"


@pytest.mark.parametrize("fmt", [4, 6])
def test_gemm_accumulate(q, orc, fmt):
    N, K, M = 96, 1024, 12
    W = (synth.q4k_matrix_np if fmt == 4 else synth.q6k_matrix_np)(SEED, 90, N, K)
    X = synth.bf16_normal_np(SEED, 91, (M, K))
    Yr, A = orc.gemm(fmt, W, N, K, X)
    Y0 = torch.randn(M, N, device="cuda")
    Y = _gemm(q, fmt, W, N, K, X, M, accumulate=True, Y0=Y0)
    base = Y0.cpu().double().numpy()
    assert (np.abs(Y - (base + Yr)) <= 1e-3 * A + 4 * 2.0 ** -24 * np.abs(base)).all()


def test_q4k_gemm_one_hot_reads_weights(q, orc):
    """x = e_k selects weight column k; the GPU's only roundings are two fp32
    multiply-adds of exact products: |y - w| <= 2^-23 (|d sc q| + |dmin m|)."""
    N, K = 64, 512
    W = synth.q4k_matrix_np(SEED, 92, N, K)
    ks = [0, 1, 2, 3, 31, 32, 63, 64, 100, 255, 256, 300, 511, 444, 77, 190]
    X = np.zeros((16, K), np.uint16)
    for r, k in enumerate(ks):
        X[r, k] = 0x3F80
    Y = _gemm(q, 4, W, N, K, X, 16)
    w = orc.dequant(4, W, N, K)
    bound = np.zeros((N, K))
    blocks = W.reshape(N, K // 256, 144)
    for n in range(N):
        for b in range(K // 256):
            qq, sc, m, d, dmin = orc.q4k_decode(blocks[n, b])
            dd, dm = orc.half_to_double(d), orc.half_to_double(dmin)
            bound[n, 256 * b:256 * (b + 1)] = np.abs(dd * np.repeat(sc, 32) * qq) + np.abs(dm * np.repeat(m, 32))
    for r, k in enumerate(ks):
        assert (np.abs(Y[r] - w[:, k]) <= 2.0 ** -23 * bound[:, k]).all()


def test_q6k_gemm_one_hot_reads_weights(q, orc):
    N, K = 48, 768
    W = synth.q6k_matrix_np(SEED, 93, N, K)
    ks = [0, 15, 16, 64, 127, 128, 255, 256, 511, 767]
    X = np.zeros((len(ks), K), np.uint16)
    for r, k in enumerate(ks):
        X[r, k] = 0x3F80
    Y = _gemm(q, 6, W, N, K, X, len(ks))
    w = orc.dequant(6, W, N, K)
    for r, k in enumerate(ks):
        assert (np.abs(Y[r] - w[:, k]) <= 2.0 ** -24 * np.abs(w[:, k])).all()


def test_q6k_gemm_one_hot_signed_scales(q, orc):
    """Signed int8 scales over the whole range: the operand sc*(q-32) is exact in
    fp16 up to 2048 in magnitude and within half an ulp (2^-11 relative) above it,
    so |y - w| <= (2^-11 + 2^-24) |w|."""
    N, K = 48, 768
    W = synth.q6k_matrix_np(SEED, 96, N, K, signed=True)
    ks = [0, 15, 16, 64, 127, 128, 255, 256, 511, 767]
    X = np.zeros((len(ks), K), np.uint16)
    for r, k in enumerate(ks):
        X[r, k] = 0x3F80
    Y = _gemm(q, 6, W, N, K, X, len(ks))
    w = orc.dequant(6, W, N, K)
    for r, k in enumerate(ks):
        assert (np.abs(Y[r] - w[:, k]) <= (2.0 ** -11 + 2.0 ** -24) * np.abs(w[:, k])).all()


def test_gemm_rows_are_independent(q, orc):
    """Row r of a 12-row product equals the 1-row product on row r (within tolerance)."""
    N, K = 200, 2048
    W = synth.q4k_matrix_np(SEED, 94, N, K)
    X = synth.bf16_normal_np(SEED, 94, (12, K))
    Y = _gemm(q, 4, W, N, K, X, 12)
    _, A = orc.gemm(4, W, N, K, X)
    for r in (0, 5, 11):
        Y1 = _gemm(q, 4, W, N, K, X[r:r + 1], 1)
        assert (np.abs(Y1[0] - Y[r]) <= 2e-3 * A[r]).all()


def test_gemm_extreme_activation_ranges(q, orc):
    """Rows far outside fp16's range still go through exactly (power-of-two row scale)."""
    N, K, M = 64, 1024, 4
    W = synth.q4k_matrix_np(SEED, 95, N, K)
    X = synth.bf16_normal_np(SEED, 95, (M, K)).astype(np.float64)
    base = synth.bf16_normal_np(SEED, 95, (M, K))
    scaled = []
    for r, s in enumerate([1e30, 1e-30, 3e4, 1.0]):
        v = orc.bf16_array_to_f64(base[r]) * s
        scaled.append(synth.bf16_bits_np(v.astype(np.float32)))
    X = np.stack(scaled)
    Yr, A = orc.gemm(4, W, N, K, X)
    Y = _gemm(q, 4, W, N, K, X, M)
    assert (np.abs(Y - Yr) <= 1e-3 * A).all()


def test_gemm_full_size_down_projection(q, orc):
    """The Q6_K-like down projection: N=5120, K=17408, 12 rows, all outputs."""
    N, K, M = 5120, 17408, 12
    g = synth.torch_gen(SEED, "cuda", 3)
    Wg = synth.q6k_matrix_torch(g, N, K, "cuda")
    Xd = synth.bf16_normal_torch(g, (M, K), "cuda")
    Y = torch.zeros(M, N, device="cuda")
    q.q6k_gemm(q.q6k_pack(Wg, N, K), N, K, Xd, M, Y)
    torch.cuda.synchronize()
    Yr, A = orc.gemm(6, Wg.cpu().numpy(), N, K, _bits(Xd))
    ratio = np.abs(Y.cpu().double().numpy() - Yr) / (1e-3 * A)
    assert ratio.max() <= 1.0, ratio.max()
    assert q.device_status() == 0


def test_gemm_full_size_down_projection_signed_scales(q, orc):
    """The down projection with signed int8 sub-block scales over the whole range
    (-128..127, as real Q6_K checkpoints carry them): N=5120, K=17408, 12 rows."""
    N, K, M = 5120, 17408, 12
    g = synth.torch_gen(SEED, "cuda", 4)
    Wg = synth.q6k_matrix_torch(g, N, K, "cuda", signed=True)
    Xd = synth.bf16_normal_torch(g, (M, K), "cuda")
    Y = torch.zeros(M, N, device="cuda")
    q.q6k_gemm(q.q6k_pack(Wg, N, K), N, K, Xd, M, Y)
    torch.cuda.synchronize()
    Yr, A = orc.gemm(6, Wg.cpu().numpy(), N, K, _bits(Xd))
    ratio = np.abs(Y.cpu().double().numpy() - Yr) / (1e-3 * A)
    assert ratio.max() <= 1.0, ratio.max()
    assert q.device_status() == 0


def test_gemm_full_size_gate_up_projection(q, orc):
    """The single gate/up projection: N=17408, K=5120, 12 rows (4 agents x 3), all outputs."""
    N, K, M = 17408, 5120, 12
    g = synth.torch_gen(SEED, "cuda", 1)
    Wd = synth.q4k_matrix_torch(g, N, K, "cuda")
    Xd = synth.bf16_normal_torch(g, (M, K), "cuda")
    Y = torch.zeros(M, N, device="cuda")
    q.q4k_gemm(Wd, N, K, Xd, M, Y)
    torch.cuda.synchronize()
    W = Wd.cpu().numpy()
    X = _bits(Xd)
    Yr, A = orc.gemm(4, W, N, K, X)
    ratio = np.abs(Y.cpu().double().numpy() - Yr) / (1e-3 * A)
    assert ratio.max() <= 1.0, ratio.max()
    assert q.device_status() == 0


# ------------------------------------------------------------------ attention

def _attn_inputs(lens, n_rows, n_qh, n_kvh, seed, cap_extra=5, qscale=1.0):
    A = len(lens)
    cap = max(l + n for l, n in zip(lens, n_rows)) + cap_extra
    ars = np.concatenate([[0], np.cumsum(n_rows)]).astype(np.int32)
    M = int(ars[-1])
    Qb = synth.bf16_normal_np(SEED, 300 + seed, (M, n_qh, 128), scale=qscale)
    Kc = synth.bf16_normal_np(SEED, 400 + seed, (A, n_kvh, cap, 128))
    Vc = synth.bf16_normal_np(SEED, 500 + seed, (A, n_kvh, cap, 128))
    return Qb, Kc, Vc, np.array(lens, np.int32), ars, cap


def _check_attn(O_gpu_bits, O_ref, B, orc):
    o = orc.bf16_array_to_f64(O_gpu_bits)
    ref_b = orc.bf16_array_to_f64(orc.f64_array_to_bf16(O_ref))
    ulp_half = np.abs(O_ref) * 2.0 ** -9
    assert (np.abs(o - O_ref) <= 2e-3 * B + ulp_half + 1e-30).all(), np.max(np.abs(o - O_ref) / (2e-3 * B + ulp_half))
    num = np.linalg.norm(o - ref_b, axis=-1)
    den = np.linalg.norm(O_ref, axis=-1)
    assert (num <= 2e-3 * den + 1e-30).all(), (num / den).max()


def _run_attn(q, Qb, Kc, Vc, lens, ars, n_qh, n_kvh, cap, max_rows=None):
    M = int(ars[-1])
    max_rows = max_rows or int(max(np.diff(ars).max(), 1))
    O = torch.zeros(max(M, 1), n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.decode_attn(_to_dev_bf16(Qb), _to_dev_bf16(Kc), _to_dev_bf16(Vc), torch.from_numpy(lens).cuda(),
                  torch.from_numpy(ars).cuda(), len(lens), max_rows, cap, n_qh, n_kvh, 128, O)
    torch.cuda.synchronize()
    return _bits(O)[:M]


ATTN_CASES = [
    ([40, 0, 7, 129], [3, 3, 3, 3], 48, 8),      # 4 agents x 3 rows, 48/8 heads, short ragged caches
    ([5, 300], [1, 4], 8, 2),                    # different rows per agent
    ([0, 1, 2], [3, 0, 2], 16, 4),               # empty caches, an agent with no rows
    ([1000, 2049, 63], [3, 3, 3], 48, 8),        # several splits, tails not tile multiples
    ([17], [16], 24, 4),                         # 16 rows of one agent x 6 heads = 96 query vectors
    ([3000], [2], 4, 4),                         # group of 1 (plain multi-head)
]


@pytest.mark.parametrize("lens,n_rows,n_qh,n_kvh", ATTN_CASES)
def test_attn_parity(q, orc, lens, n_rows, n_qh, n_kvh):
    Qb, Kc, Vc, lens, ars, cap = _attn_inputs(lens, n_rows, n_qh, n_kvh, seed=len(lens) + n_qh)
    O_ref, B = orc.decode_attn(Qb, Kc, Vc, lens, ars, n_qh, n_kvh, 128, cap)
    O = _run_attn(q, Qb, Kc, Vc, lens, ars, n_qh, n_kvh, cap)
    _check_attn(O, O_ref, B, orc)


def test_attn_peaked_scores(q, orc):
    """Queries scaled x4: sharply peaked softmax."""
    Qb, Kc, Vc, lens, ars, cap = _attn_inputs([700, 90], [3, 3], 48, 8, seed=7, qscale=4.0)
    O_ref, B = orc.decode_attn(Qb, Kc, Vc, lens, ars, 48, 8, 128, cap)
    _check_attn(_run_attn(q, Qb, Kc, Vc, lens, ars, 48, 8, cap), O_ref, B, orc)


def test_attn_full_size_23k_context(q, orc):
    """4 agents x 23000 cached tokens, 3 rows each, 48 q-heads / 8 kv-heads, every output."""
    n_qh, n_kvh, A, L = 48, 8, 4, 23000
    cap = L + 3
    g = synth.torch_gen(SEED, "cuda", 2)
    Kd = synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda")
    Vd = synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda")
    Qd = synth.bf16_normal_torch(g, (12, n_qh, 128), "cuda")
    lens = np.full(A, L, np.int32)
    ars = np.arange(0, 13, 3, dtype=np.int32)
    O = torch.zeros(12, n_qh, 128, dtype=torch.bfloat16, device="cuda")
    q.decode_attn(Qd, Kd, Vd, torch.from_numpy(lens).cuda(), torch.from_numpy(ars).cuda(), A, 3, cap, n_qh, n_kvh,
                  128, O)
    torch.cuda.synchronize()
    O_ref, B = orc.decode_attn(_bits(Qd), _bits(Kd), _bits(Vd), lens, ars, n_qh, n_kvh, 128, cap)
    _check_attn(_bits(O), O_ref, B, orc)
