"""Contract identities (host code of the library, no GPU): SHA-256 digests of
the semantic, numerical-policy and deployment texts (IsoExec summary page,
"Contract Structure and Enforcement", Identities).  The library's SHA-256 is
checked against Python's hashlib, an independent implementation."""
import hashlib
import itertools

import pytest

from gated_deltanet_cpr_delta_b200 import build, gdn

KINDS = (gdn.ID_SEMANTIC, gdn.ID_NUMERICAL_POLICY, gdn.ID_DEPLOYMENT)
SHAPES = [(d, d, C) for d in (16, 32, 64, 128) for C in (16, 32, 64)]
DTYPES = list(itertools.product((gdn.GDN_F32, gdn.GDN_BF16), repeat=2))


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return gdn.load_library()


@pytest.mark.parametrize("msg", [b"", b"abc", b"abcdbcdecdefdefgefghfghighijhijkijkljklmklmnlmnomnopnopq",
                                 b"a" * 1000000, bytes(range(256)) * 5])
def test_sha256_standard_messages(msg):
    assert gdn.gdn_sha256_hex(msg) == hashlib.sha256(msg).hexdigest()


def test_sha256_every_padding_length():
    # lengths around the 55/56/64-byte padding boundaries and several blocks
    for n in range(0, 300):
        m = bytes((31 * i + n) & 0xFF for i in range(n))
        assert gdn.gdn_sha256_hex(m) == hashlib.sha256(m).hexdigest(), n


def test_identity_is_sha256_of_its_text():
    for kind, (dk, dv, C), (ti, to) in itertools.product(KINDS, SHAPES, DTYPES):
        text = gdn.gdn_contract_text(kind, dk, dv, C, ti, to)
        assert gdn.gdn_contract_identity(kind, dk, dv, C, ti, to) == hashlib.sha256(text.encode()).hexdigest()


def test_identities_tell_configurations_apart():
    seen = {}
    for kind, (dk, dv, C), (ti, to) in itertools.product(KINDS, SHAPES, DTYPES):
        ident = gdn.gdn_contract_identity(kind, dk, dv, C, ti, to)
        assert ident not in seen, (seen.get(ident), (kind, dk, C, ti, to))
        seen[ident] = (kind, dk, C, ti, to)


def test_policy_and_deployment_texts_name_what_they_pin():
    pol = gdn.gdn_contract_text(gdn.ID_NUMERICAL_POLICY, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_BF16)
    assert f"contract={gdn.gdn_contract_id()}" in pol
    for needle in ("8 leaves", "round to nearest even", "tcgen05.mma kind::tf32", "mma.sync.m16n8k8",
                   "d_k=128 d_v=128 C=64 in=bf16 out=bf16"):
        assert needle in pol
    dep = gdn.gdn_contract_text(gdn.ID_DEPLOYMENT, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_BF16)
    assert f"kernel_sources_sha256={build.sources_sha256()}" in dep
    assert "target=sm_100a" in dep
    sem = gdn.gdn_contract_text(gdn.ID_SEMANTIC, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_BF16)
    assert "S_t = alpha_t * S_{t-1} * (I - beta_t * k_t * k_t^T) + beta_t * v_t * k_t^T" in sem


def test_text_buffer_contract(lib):
    import ctypes
    n = lib.gdn_contract_text(1, 64, 64, 32, 0, 0, None, 0)
    assert n > 0
    small = ctypes.create_string_buffer(10)
    assert lib.gdn_contract_text(1, 64, 64, 32, 0, 0, small, 10) == n   # truncated, full length returned
    assert len(small.value) == 9
    assert lib.gdn_contract_text(1, 64, 64, 32, 0, 0, None, 5) == -1    # NULL with a capacity


def test_rejects_unsupported_and_bad_kind(lib):
    import ctypes
    out = ctypes.create_string_buffer(65)
    assert lib.gdn_contract_identity(1, 24, 24, 64, 1, 1, out) == 2      # head dim not compiled in
    assert lib.gdn_contract_identity(1, 128, 64, 64, 1, 1, out) == 2     # d_k != d_v
    assert lib.gdn_contract_identity(1, 128, 128, 48, 1, 1, out) == 2    # chunk size
    assert lib.gdn_contract_identity(1, 128, 128, 64, 5, 1, out) == 2    # dtype
    assert lib.gdn_contract_identity(7, 128, 128, 64, 1, 1, out) == 1    # kind
    assert lib.gdn_contract_identity(1, 128, 128, 64, 1, 1, None) == 1
    assert lib.gdn_contract_text(7, 128, 128, 64, 1, 1, None, 0) == -1
    assert lib.gdn_sha256_hex(None, 3, out) == 1
