"""The C-ABI library: builds for sm_100a, loads, and exports every declared call.
No compute is launched here (these tests run without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

import audio_encoder_tower_b200 as E
from audio_encoder_tower_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"ENC_API\s+[\w\s\*]*?\b(enc_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return E.load_library()


def test_headers_declare_the_boundary():
    names = declared_symbols()
    for n in ("enc_create", "enc_forward", "enc_destroy", "enc_get_status", "enc_output_positions",
              "enc_status_string"):
        assert n in names
    assert names == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_library_is_sm100a(lib):
    # the shared object embeds an sm_100a image: nvcc was given compute_100a/sm_100a
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)
    assert os.path.getsize(build.LIB) > 100_000


def test_status_strings(lib):
    assert E.status_string(0) == "ok"
    assert "sm_100" in E.status_string(2)
    assert E.status_string(99) == "unknown status"


def test_config_struct_matches_header():
    src = open(os.path.join(ROOT, "include", "enc.h")).read()
    body = src[src.index("typedef struct enc_config"):src.index("} enc_config;")]
    fields = re.findall(r"\b(?:int32_t|uint32_t|float)\s+(\w+);", body)
    assert fields == [f for f, _ in binding.EncConfig._fields_]
    wbody = src[src.index("typedef struct enc_weights"):src.index("} enc_weights;")]
    wfields = re.findall(r"\*(?:const \*)?(\w+)", wbody)
    assert wfields == [f for f, _ in binding.EncWeights._fields_]
