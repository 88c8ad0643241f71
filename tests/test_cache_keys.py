"""The oracle cache's keys: they follow what the oracle sources compute, not their documentation."""
import os

import helpers


def _digest_of(tmp_path, src):
    p = tmp_path / "m.py"
    p.write_text(src)
    return helpers._code_of(str(p))


def test_docstring_and_comment_edits_keep_the_key(tmp_path):
    a = _digest_of(tmp_path, '"""Module doc."""\n\ndef f(x):\n    """Doc."""\n    return x + 1  # note\n')
    b = _digest_of(tmp_path, '"""Other words."""\n\ndef f(x):\n    """Changed."""\n    # a comment\n    return x + 1\n')
    assert a == b


def test_code_edits_change_the_key(tmp_path):
    a = _digest_of(tmp_path, 'def f(x):\n    """Doc."""\n    return x + 1\n')
    b = _digest_of(tmp_path, 'def f(x):\n    """Doc."""\n    return x + 2\n')
    c = _digest_of(tmp_path, 'def f(x):\n    return x + 1\n')   # only the docstring removed
    assert a != b and a == c


def test_the_oracle_digest_covers_the_oracle_and_the_input_generator():
    root = helpers.ROOT
    assert os.path.exists(os.path.join(root, "oracle/mate_oracle.py"))
    d0 = helpers._oracle_digest(())
    assert d0 != helpers._oracle_digest(("tests/bf16_floor.py",))
    assert len(d0) == 16
