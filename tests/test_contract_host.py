"""Contract digests of the CPR region (host only; no GPU needed).

"NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
section "The execution contract": three SHA-256 identity digests (semantic
equivalence, numerical policy, deployment settings that do not affect bits),
and engines whose numerical policies differ refuse to run together.
"""
import hashlib
import random

import pytest
import torch

from rl_train_numerics_b200 import _abi as gdn

KINDS = [gdn.GDN_DIGEST_SEMANTIC, gdn.GDN_DIGEST_POLICY, gdn.GDN_DIGEST_DEPLOYMENT]
SHAPES = [  # (in_dtype, out_dtype, d) the library runs
    (torch.bfloat16, torch.bfloat16, 128), (torch.bfloat16, torch.float32, 128),
    (torch.bfloat16, torch.bfloat16, 64), (torch.float32, torch.float32, 64),
    (torch.float32, torch.bfloat16, 64),
]


# Example digests published with the SHA-256 definition (FIPS 180-2, appendix B).
@pytest.mark.parametrize("msg,hexdigest", [
    (b"abc", "ba7816bf8f01cfea414140de5dae2223b00361a396177a9cb410ff61f20015ad"),
    (b"abcdbcdecdefdefgefghfghighijhijkijkljklmklmnlmnomnopnopq",
     "248d6a61d20638b8e5c026930c3e6039a33ce45964ff2167f6ecedd419db06c1"),
    (b"a" * 1000000, "cdc76e5c9914fb9281a1c7e284d73e67f1809a48a497200e046d39ccc7112cd0"),
    (b"", "e3b0c44298fc1c149afbf4c8996fb92427ae41e4649b934ca495991b7852b855"),
])
def test_sha256_published_examples(msg, hexdigest):
    assert gdn.sha256(msg).hex() == hexdigest


def test_sha256_every_length_across_padding_boundaries():
    rng = random.Random(5)
    for n in range(0, 300):
        msg = bytes(rng.randrange(256) for _ in range(n))
        assert gdn.sha256(msg) == hashlib.sha256(msg).digest(), n


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("in_dt,out_dt,d", SHAPES)
def test_digest_is_sha256_of_descriptor(kind, in_dt, out_dt, d):
    text = gdn.contract_descriptor(kind, in_dt, out_dt, d, d)
    assert text.startswith("gdn-cpr contract descriptor v1\n")
    assert gdn.contract_digest(kind, in_dt, out_dt, d, d) == hashlib.sha256(text.encode()).digest()


def test_policy_separates_what_moves_bits_semantic_does_not():
    pol = {s: gdn.contract_digest(gdn.GDN_DIGEST_POLICY, *s[:2], s[2], s[2]) for s in SHAPES}
    assert len(set(pol.values())) == len(SHAPES)  # every dtype / size pair has its own policy
    sem = lambda i, o, d: gdn.contract_digest(gdn.GDN_DIGEST_SEMANTIC, i, o, d, d)
    # the same computation whatever the dtypes: one semantic digest per (d, C)
    assert sem(torch.bfloat16, torch.bfloat16, 64) == sem(torch.float32, torch.float32, 64)
    assert sem(torch.bfloat16, torch.bfloat16, 64) != sem(torch.bfloat16, torch.bfloat16, 128)
    text = gdn.contract_descriptor(gdn.GDN_DIGEST_POLICY, torch.bfloat16, torch.bfloat16, 128, 128)
    for key in ("step_schedule=", "boundary_schedule=", "walk=tcgen05", "compile=", "splits=",
                "backward="):
        assert key in text
    assert "gradients=" in gdn.contract_descriptor(gdn.GDN_DIGEST_SEMANTIC, torch.bfloat16,
                                                   torch.bfloat16, 128, 128)
    text64 = gdn.contract_descriptor(gdn.GDN_DIGEST_POLICY, torch.bfloat16, torch.bfloat16, 64, 64)
    assert "walk=mma.sync" in text64


def test_check_accepts_own_policy_and_refuses_others():
    mine = gdn.contract_digest(gdn.GDN_DIGEST_POLICY, torch.bfloat16, torch.bfloat16, 128, 128)
    assert gdn.contract_check(mine, torch.bfloat16, torch.bfloat16, 128, 128) == gdn.GDN_OK
    assert gdn.contract_check(mine, torch.bfloat16, torch.float32, 128, 128) == gdn.GDN_ERR_CONTRACT
    assert gdn.contract_check(mine, torch.bfloat16, torch.bfloat16, 64, 64) == gdn.GDN_ERR_CONTRACT
    flipped = bytes([mine[0] ^ 1]) + mine[1:]
    assert gdn.contract_check(flipped, torch.bfloat16, torch.bfloat16, 128, 128) == \
        gdn.GDN_ERR_CONTRACT
    sem = gdn.contract_digest(gdn.GDN_DIGEST_SEMANTIC, torch.bfloat16, torch.bfloat16, 128, 128)
    assert gdn.contract_check(sem, torch.bfloat16, torch.bfloat16, 128, 128) == gdn.GDN_ERR_CONTRACT
    assert gdn.status_string(gdn.GDN_ERR_CONTRACT).startswith("GDN_ERR_CONTRACT")


def test_contract_rejects_on_host():
    L = gdn.lib
    out = bytes(32)
    assert L.gdn_cpr_contract_digest(7, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 64, out) == \
        gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_cpr_contract_digest(1, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 64, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_cpr_contract_digest(1, gdn.GDN_F32, gdn.GDN_BF16, 128, 128, 64, out) == \
        gdn.GDN_ERR_UNSUPPORTED  # fp32 inputs only at d = 64
    assert L.gdn_cpr_contract_digest(1, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 32, out) == \
        gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_cpr_contract_check(None, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 64) == \
        gdn.GDN_ERR_INVALID_ARG
    n = __import__("ctypes").c_size_t(0)
    assert L.gdn_cpr_contract_descriptor(1, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 64, None, 0,
                                         __import__("ctypes").byref(n)) == gdn.GDN_OK
    small = __import__("ctypes").create_string_buffer(8)
    assert L.gdn_cpr_contract_descriptor(1, gdn.GDN_BF16, gdn.GDN_BF16, 128, 128, 64, small, 8,
                                         None) == gdn.GDN_ERR_INVALID_ARG
